"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

The path shards into independent replicas (one seeded batch per rank, no
data-path collective); only the timing reduction crosses ranks.  These tests
run the same reduction and bookkeeping over gloo on CPU.
"""
import json
import os
import socket
import subprocess
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from workloads import WORKLOADS, make_inputs
        w = WORKLOADS["tiny_L256_D64"]
        local_ms = [10.0, 25.0][rank]
        m = bench.max_over_ranks(local_ms, world)
        seed = bench.rank_seed(w, rank)
        q, _, _ = make_inputs(w, device="cpu", seed=seed)
        # gather the replicas' first values to check they differ
        t = torch.tensor([float(q.flatten()[0])])
        gathered = [torch.zeros(1) for _ in range(world)]
        dist.all_gather(gathered, t)
        out[rank] = (m, seed, [float(g) for g in gathered],
                     bench.job_tflops(1e12, world, 4, m))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_reduction_and_replicas():
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(2, port, out), nprocs=2, start_method="spawn", join=True)
    r0, r1 = out[0], out[1]
    assert r0[0] == r1[0] == 25.0                 # max over ranks
    assert r0[1] != r1[1]                         # distinct seeds per rank
    assert r0[2] == r1[2] and r0[2][0] != r0[2][1]  # distinct replica inputs
    # weak scaling: 2 ranks x 4 steps x 1 TFLOP over the slowest rank's 25 ms
    assert abs(r0[3] - 2 * 4 * 1e12 / 0.025 / 1e12) < 1e-9


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0", "--workload", "tiny_L256_D64"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_line_on_rank_zero():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0", "--workload", "tiny_L256_D64",
                        "--cpu-budget", "1"], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    d = json.loads(r.stdout.strip().splitlines()[-1])
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
