"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

The path shards into independent replicas (one seeded batch per rank) or into
kv-head slices of one batch, with no data-path collective either way; only the
timing reduction crosses ranks.  These tests run the same reduction, the head
ranges and the rank bookkeeping over gloo on CPU, and start bench.py's own
launcher (its reference arm, which needs no GPU).
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


def _shard_worker(rank, world, port, out):
    """Each rank takes its kv-head range of one batch (bench --shard heads) and
    the ranks check over gloo that the ranges are disjoint and cover every head."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from workloads import WORKLOADS, make_inputs
        w = WORKLOADS["tiny_L256_D64"].with_(Hq=8, Hkv=4, L=64)
        g0, g1 = bench.shard_heads(w.Hkv, world, rank)
        ranges = [torch.zeros(2, dtype=torch.int64) for _ in range(world)]
        dist.all_gather(ranges, torch.tensor([g0, g1]))
        # every rank draws the same batch in head-shard mode
        q, k, _ = make_inputs(w, device="cpu", seed=bench.rank_seed(w, rank, "heads"))
        G = w.Hq // w.Hkv
        part = q[:, g0 * G:g1 * G].contiguous()
        sums = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(sums, part.double().sum().reshape(1))
        out[rank] = ([tuple(int(x) for x in r) for r in ranges], [float(x) for x in sums],
                     float(q.double().sum()))
    finally:
        dist.destroy_process_group()


def test_two_rank_head_shards_cover_the_batch():
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.start_processes(_shard_worker, args=(2, port, out), nprocs=2, start_method="spawn",
                       join=True)
    ranges0, sums0, total0 = out[0]
    ranges1, sums1, total1 = out[1]
    assert ranges0 == ranges1 == [(0, 2), (2, 4)]
    assert total0 == total1                       # the same batch on both ranks
    assert abs(sum(sums0) - total0) < 1e-6 * max(1.0, abs(total0))


def test_shard_heads_ranges():
    import bench
    for hkv in (1, 2, 3, 8, 16):
        for world in range(1, hkv + 1):
            r = [bench.shard_heads(hkv, world, i) for i in range(world)]
            assert r[0][0] == 0 and r[-1][1] == hkv
            assert all(a[1] == b[0] for a, b in zip(r, r[1:]))
            sizes = [g1 - g0 for g0, g1 in r]
            assert min(sizes) >= 1 and max(sizes) - min(sizes) <= 1
    import pytest
    with pytest.raises(ValueError):
        bench.shard_heads(8, 16, 0)


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
                        "--gpus", "2", "--steps", "1", "--warmup", "0", "--workload",
                        "tiny_L256_D64"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_gpus_must_match_world_size():
    """Under a launcher that set WORLD_SIZE, --gpus must name the same count."""
    env = dict(os.environ, RANK="0", WORLD_SIZE="2", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "4", "--steps", "1", "--warmup", "0", "--workload",
                        "tiny_L256_D64"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode != 0 and "WORLD_SIZE" in r.stderr


def test_gpus_without_launcher_starts_the_ranks():
    """--gpus 2 without a launcher: bench.py starts two ranks itself (torchrun
    on 127.0.0.1) and the line rank 0 prints counts both."""
    env = {k_: v_ for k_, v_ in os.environ.items()
           if k_ not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0", "--workload",
                        "tiny_L256_D64", "--cpu-budget", "1"],
                       capture_output=True, text=True, env=env, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [x for x in r.stdout.strip().splitlines() if x.startswith("{")]
    assert len(lines) == 1
    assert json.loads(lines[0])["n_gpus"] == 2


def test_reference_arm_line_on_rank_zero():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0", "--workload", "tiny_L256_D64",
                        "--cpu-budget", "1"], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    d = json.loads(r.stdout.strip().splitlines()[-1])
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
