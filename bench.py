"""Benchmark: fused YaRN-RoPE causal attention prefill on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step = one pass of the hot path over one batch of the workload, one
lcx_attn_fwd call: the RoPE table for the mode (host), the rotate pass over the
keys into a buffer (args.k_rot: every key rotated once, mscale included), and
the fused kernel (queries rotated on chip, QK^T, online softmax, PV).  In the
split-QK^T mode the pass writes the keys' fp16 and 8-bit cross parts.  Prints ONE
JSON line (rank 0).

* value      : attention TFLOP/s, algorithmic FLOPs = 4 * D * (visible query/key
               pairs) * B * Hq summed over all ranks, divided by the max over ranks
               of the device time of K steps (CUDA events, inputs resident in HBM).
* e2e        : the same metric through attn_fwd_host (pinned host q/k/v copied in,
               o copied out, inside the timed region).
* roofline   : the attention kernel against the measured dense BF16 peak.
* cpu_baseline: the fp64 CPU oracle on a bounded sample of the same workload.
* --impl reference: the oracle alone, as the reference arm (rank 0 only).

* configs    : every workload of workloads.WORKLOADS measured the same way (one
               lcx_attn_fwd call per step, inputs resident in HBM, L2 flushed
               between calls whose inputs fit in L2): attention TFLOP/s and its
               fraction of the sustained and burst bf16 peaks, the mean call
               time, apply_rope GB/s against HBM, the tiny workload's latency,
               and the oracle's extrapolated full-size CPU time (an estimate).

Multi-GPU: `--gpus N` with N > 1 runs N ranks, one per GPU (started with
torchrun by this script when it was not launched under torchrun itself; under
torchrun WORLD_SIZE must equal N).  `--shard replicas` (default): every rank
runs an independent replica (its own seeded batch) -- the path has no exchange
step, so there is no data-path collective and scaling is weak.  `--shard heads`:
the ranks split one batch's kv heads (rank r takes kv heads
[r Hkv / N, (r + 1) Hkv / N) and their query heads, and writes that slice of
O), again with no data-path collective; the total work is fixed, so scaling is
strong.  The NCCL process group carries only the barriers and the max-over-ranks
timing.  The headline inputs are larger than L2 (126 MB), so no flush is needed.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from workloads import HEADLINE, WORKLOADS, attn_flops, make_inputs, rope_bytes, \
    visible_pairs  # noqa: E402

METRIC = "fused YaRN-RoPE causal attention prefill TFLOP/s and % dense BF16 peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one attention
# launch on the headline workload (yarn_L131072_s16), from a one-pass ncu capture
# of the current kernel (keys pre-rotated by the rotate pass); None until the
# current kernel has been captured.  Only valid for that workload.
ATTN_TRAFFIC_BYTES = {"yarn_L131072_s16": 2987733248 + 1077540864}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms while running."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=2)

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        loaded = [s for s in sm if s >= 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    """The largest of the ranks' values (device times are reported as the max)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(w, rank, shard="replicas"):
    """Replicas: each rank runs an independent replica of the workload with its
    own seed.  Head shards: every rank draws the same batch (the workload's seed)
    and keeps its slice of the heads."""
    return w.seed if shard == "heads" else w.seed + rank


def shard_heads(Hkv, world, rank):
    """The kv heads [g0, g1) rank `rank` of `world` takes when the ranks split
    one batch by heads (its query heads are [g0 G, g1 G)).  Contiguous, disjoint,
    covering every kv head; sizes differ by at most one."""
    if not 1 <= world <= Hkv:
        raise ValueError("cannot split %d kv heads over %d ranks" % (Hkv, world))
    return rank * Hkv // world, (rank + 1) * Hkv // world


def job_tflops(flops_per_rank, world, steps, max_ms):
    """Whole-job throughput: the work of all ranks over the slowest rank's time."""
    return flops_per_rank * world * steps / (max_ms * 1e-3) / 1e12


# ------------------------------------------------------------------ oracle
def oracle_sample(w, budget_s=15.0, seed=0):
    """Time the fp64 oracle on a bounded sample of the workload: one (batch, kv
    head) with its query heads, rows taken from the end of the sequence (the
    heaviest rows).  Returns (TFLOP/s, seconds, threads, description)."""
    import oracle
    g = torch.Generator().manual_seed(seed)
    L, D = w.L, w.D
    k = torch.randn((1, 1, L, D), generator=g).to(w.torch_dtype).float().numpy()
    v = torch.randn((1, 1, L, D), generator=g).to(w.torch_dtype).float().numpy()
    G = w.Hq // w.Hkv
    table, ms, _ = oracle.rope_table(w.mode, D, w.base, w.scale, w.original_max_pos,
                                     w.alpha, w.beta)
    nthreads = oracle.num_threads(0)
    scale = w.softmax_scale if w.softmax_scale > 0 else None
    # calibrate with a few rows, then size the sample to the time budget
    n_rows = 2 * nthreads
    while True:
        rows = np.arange(L - n_rows, L) % L
        heads = np.arange(n_rows) % G
        q = torch.randn((n_rows, D), generator=g).to(w.torch_dtype).float().numpy()
        t0 = time.perf_counter()
        oracle.attn_rows(q, np.zeros(n_rows), heads, rows, k, v, G, table, ms, w.pairing, 0,
                         w.causal, w.window, w.sinks, scale, 0)
        dt = time.perf_counter() - t0
        flops = sum(4 * D * _row_visible(w, int(i)) for i in rows)
        if dt >= budget_s / 3 or n_rows >= 1 << 16:
            break
        n_rows = int(min(n_rows * max(2.0, budget_s / max(dt, 1e-3) * 0.5), 1 << 16))
    desc = ("fp64 oracle, 1 kv head of %s: %d query rows (the last %d positions, %d query "
            "heads) incl. rotating all %d keys" % (w.name, n_rows, n_rows, G, L))
    return flops / dt / 1e12, dt, nthreads, desc


def _row_visible(w, i):
    if not w.causal:
        return w.L
    n = i + 1
    if w.window > 0 and i - w.window + 1 > 0:
        lo = i - w.window + 1
        n = w.window + min(w.sinks, lo)
    return n


# ------------------------------------------------------------------ GPU arm
def bench_gpu(args, world, rank, local):
    import ntk_rope_flashattn_b200 as lcx
    w = WORKLOADS[args.workload]
    if args.batch > 0:
        w = w.with_(B=args.batch)
    dev = torch.device("cuda", local)
    q, k, v = make_inputs(w, device=dev, seed=rank_seed(w, rank, args.shard))
    g0, g1 = 0, w.Hkv
    if args.shard == "heads":
        G = w.Hq // w.Hkv
        g0, g1 = shard_heads(w.Hkv, world, rank)
        q, k, v = (q[:, g0 * G:g1 * G].contiguous(), k[:, g0:g1].contiguous(),
                   v[:, g0:g1].contiguous())
        torch.cuda.empty_cache()
    rope = lcx.RopeParams(w.mode, w.D, w.base, w.scale, w.original_max_pos, w.alpha, w.beta,
                          w.pairing)
    o = torch.empty_like(q)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    # keys rotated once per step into k_rot (split-QK^T with bf16 keys: fp16 parts, then
    # 8-bit cross parts of as many bytes, then V in fp16)
    rotate_once = True
    parts = 3 if (w.split_qk and k.dtype == torch.bfloat16) else 1
    k_rot = torch.empty((parts,) + tuple(k.shape), dtype=k.dtype, device=dev)
    kw = dict(causal=w.causal, window=w.window, sinks=w.sinks, softmax_scale=w.softmax_scale,
              split_qk=w.split_qk, out=o, status=status, k_rot=k_rot)
    stream = torch.cuda.current_stream(dev)

    def step():
        lcx.attn_fwd(q, k, v, rope, **kw)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert int(status.item()) == 0, "device watchdog fired during warm-up"

    # --- device-timed steps (per-launch events on the launching stream)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for i in range(args.steps):
            evs[i][0].record(stream)
            step()
            evs[i][1].record(stream)
        end.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    total_ms = start.elapsed_time(end)
    launch_ms = [a.elapsed_time(b) for a, b in evs]
    assert int(status.item()) == 0, "device watchdog fired"
    total_ms = max_over_ranks(total_ms, world)
    flops_rank = attn_flops(w) * (g1 - g0) // w.Hkv
    # whole-job work: all replicas, or the one batch the head shards split
    flops_job = attn_flops(w) if args.shard == "heads" else flops_rank * world
    tflops = flops_job * args.steps / (total_ms * 1e-3) / 1e12

    # --- the same step with every K tile rotated on chip by each CTA that reads
    # it (no key buffer): the kernel-only variant of the path, for comparison
    kw_chip = dict(kw, k_rot=None)
    for _ in range(2):
        lcx.attn_fwd(q, k, v, rope, **kw_chip)
    torch.cuda.synchronize()
    a_ev, b_ev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps_chip = max(2, min(args.steps, 3))
    a_ev.record(stream)
    for _ in range(reps_chip):
        lcx.attn_fwd(q, k, v, rope, **kw_chip)
    b_ev.record(stream)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, "device watchdog fired (keys rotated on chip)"
    chip_ms = a_ev.elapsed_time(b_ev) / reps_chip
    chip_tflops = flops_rank / (chip_ms * 1e-3) / 1e12

    # --- apply_rope (the unfused rotate-pairs pass) on Q and K, for its own roofline
    qr, kr = torch.empty_like(q), torch.empty_like(k)
    for _ in range(3):
        lcx.apply_rope(q, rope, out=qr)
        lcx.apply_rope(k, rope, out=kr)
    torch.cuda.synchronize()
    rope_ev = []
    for _ in range(max(3, args.steps)):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        lcx.apply_rope(q, rope, out=qr)
        lcx.apply_rope(k, rope, out=kr)
        b.record(stream)
        rope_ev.append((a, b))
    torch.cuda.synchronize()
    rope_ms = statistics.median(a.elapsed_time(b) for a, b in rope_ev)
    # the keys' rotate pass alone (part of every step when rotate_once)
    k_ev = []
    for _ in range(max(3, args.steps)):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        lcx.apply_rope(k, rope, out=kr)
        b.record(stream)
        k_ev.append((a, b))
    torch.cuda.synchronize()
    k_rope_ms = statistics.median(a.elapsed_time(b) for a, b in k_ev) if rotate_once else 0.0
    del qr, kr

    # --- split-KV decode: one new token per query head against the whole cache
    extras = world == 1 and not args.no_extras
    decode = bench_decode(lcx, w, q, k, v, rope, stream, status) if extras else None
    mla = bench_mla(lcx, dev, stream, status) if extras else None

    # --- end to end through host buffers
    qh, kh, vh = (t.cpu().pin_memory() for t in (q, k, v))
    ws = {}
    for _ in range(max(1, min(args.warmup, 2))):
        lcx.attn_fwd_host(qh, kh, vh, rope, device=dev, workspace=ws, causal=w.causal,
                          window=w.window, sinks=w.sinks, softmax_scale=w.softmax_scale,
                          split_qk=w.split_qk, rotate_k_once=rotate_once)
    torch.cuda.synchronize()
    barrier(world)
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_start.record(stream)
    for _ in range(args.steps):
        oh = lcx.attn_fwd_host(qh, kh, vh, rope, device=dev, workspace=ws, causal=w.causal,
                               window=w.window, sinks=w.sinks, softmax_scale=w.softmax_scale,
                               split_qk=w.split_qk, rotate_k_once=rotate_once)
    e_end.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e_start.elapsed_time(e_end), world)
    e2e_tflops = flops_job * args.steps / (e2e_ms * 1e-3) / 1e12
    h2d = sum(t.numel() * t.element_size() for t in (qh, kh, vh))
    d2h = oh.numel() * oh.element_size()
    del qh, kh, vh, ws

    peaks, peak_src = load_peaks()
    # the attention kernel's own time: the step minus the keys' rotate pass
    avg_launch = statistics.mean(launch_ms) - k_rope_ms
    achieved = flops_rank / (avg_launch * 1e-3) / 1e12
    peak = float(peaks["bf16_tflops_sustained"])
    rope_gbs = rope_bytes(w) / (rope_ms * 1e-3) / 1e9
    res = {
        "metric": METRIC,
        "value": round(tflops, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(total_ms / args.steps, 3),
        "higher_is_better": True,
        "scaling": "strong" if args.shard == "heads" else "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": ("synthetic (seeded N(0,1) q/k/v, seed 0, kv heads split over the ranks)"
                 if args.shard == "heads" else "synthetic (seeded N(0,1) q/k/v, seed 0 + rank)"),
        "impl": "lcx",
        "config": {
            "workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "L": w.L, "D": w.D,
            "rope": w.mode, "scale": w.scale, "original_max_pos": w.original_max_pos,
            "alpha": w.alpha, "beta": w.beta, "causal": w.causal, "window": w.window,
            "sinks": w.sinks, "split_qk": w.split_qk, "visible_pairs_per_head": visible_pairs(w.L, w.causal, w.window,
                                                                      w.sinks),
            "flops_per_step_per_gpu": flops_rank,
            "l2": "inputs larger than L2 (q+k+v = %.2f GB), no flush" % (
                sum(t.numel() * t.element_size() for t in (q, k, v)) / 1e9),
            "parallelism": ("heads sharded over %d ranks (rank r: kv heads [r Hkv/N, (r+1) "
                            "Hkv/N) and their query heads), no data-path collective" % world
                            if args.shard == "heads" else
                            "replicas x%d (independent batches, no collective)" % world),
            "flops_per_step_job": flops_job,
        },
        "gpu_launches": args.steps * (2 if rotate_once else 1),
        "roofline": {
            "bound": "tensor", "achieved": round(achieved, 2), "peak": peak,
            "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
            "peak_kind": "bf16_tflops_sustained of %s" % peak_src,
            "frac_of_burst": round(achieved / float(peaks["bf16_tflops"]), 4),
            "traffic": ATTN_TRAFFIC_BYTES.get(w.name),
            "algorithmic_bytes": (sum(t.numel() * t.element_size() for t in (q, k, v))
                                  + o.numel() * o.element_size()),
            "kernel": "attn_fwd_kernel", "avg_launch_ms": round(avg_launch, 3),
            "k_rotate_pass_ms": round(k_rope_ms, 4),
            "launch_ms": [round(x, 3) for x in launch_ms],
        },
        "apply_rope": {
            "bound": "hbm", "bytes": rope_bytes(w), "ms": round(rope_ms, 4),
            "achieved": round(rope_gbs, 1), "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
            "frac": round(rope_gbs / float(peaks["hbm_gbs"]), 4),
        },
        "e2e": {"value": round(e2e_tflops, 2), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "clocks": clk.summary(),
        "keys_rotated_on_chip": {
            "what": "the same step without a key buffer: every K tile rotated in shared "
                    "memory by each CTA that reads it (the single-kernel variant)",
            "ms_per_step": round(chip_ms, 3), "value": round(chip_tflops, 2),
            "unit": "TFLOP/s", "launches_per_step": 1, "steps": reps_chip},
        "splitkv_decode": decode,
        "mla_prefill": mla,
    }
    if mla is not None:
        mla["peak"] = float(peaks["bf16_tflops_sustained"])
        mla["frac"] = round(mla["achieved"] / mla["peak"], 4)
    if decode is not None:
        decode["peak"] = float(peaks["hbm_gbs"])
        decode["frac"] = round(decode["achieved"] / decode["peak"], 4)
        res["gpu_launches_decode"] = decode["launches"]
    del q, k, v, o
    torch.cuda.empty_cache()
    if extras and not args.no_configs:
        res["configs"] = bench_configs(lcx, dev, stream, status, peaks, local)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        val, secs, cores, desc = oracle_sample(w, budget_s=args.cpu_budget)
        res["cpu_baseline"] = {"value": val, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                               "sample": desc, "seconds": round(secs, 2)}
        if "configs" in res:
            oracle_estimates(res["configs"], budget_s=args.cpu_budget_per_config)
    return res


L2_BYTES = 126 * 1024 * 1024


def _call_ms(fn, stream, reps, flush=None, warm=2, per_call=False):
    """Device time of one fn() (CUDA events on the launching stream): the mean
    over reps back-to-back calls, or, with `flush` or `per_call`, the median of
    reps calls each timed alone.  With `flush` (a buffer larger than L2) the
    buffer is rewritten before every call, so no call finds the previous one's
    data in L2."""
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    if flush is None and not per_call:
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps
    evs = []
    for _ in range(reps):
        if flush is not None:
            flush.add_(1)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        evs.append((a, b))
    torch.cuda.synchronize()
    return statistics.median(a.elapsed_time(b) for a, b in evs)


def _graph_and_host_us(fn, n=50):
    """A launch-bound call measured two more ways: the host time to issue one
    call (no synchronisation in between), and the device time per call when n
    calls captured once into a CUDA graph are replayed (no host work between
    the launches)."""
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for _ in range(n):
        fn()
    host_us = (time.perf_counter() - t0) / n * 1e6
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        for _ in range(n):
            fn()
    g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    cur = torch.cuda.current_stream()
    a.record(cur)
    g.replay()
    b.record(cur)
    torch.cuda.synchronize()
    graph_us = a.elapsed_time(b) / n * 1e3
    del g
    return graph_us, host_us


def bench_configs(lcx, dev, stream, status, peaks, local, reps=10):
    """Every workload measured like the headline: one lcx_attn_fwd call per
    step (host table, the keys' rotate pass into a buffer, the attention kernel),
    inputs resident in HBM; the median of `reps` calls, each timed alone.
    Workloads whose inputs fit in L2 have L2 flushed before every call.  The
    tiny workload is launch-bound: its number is the latency of one call (mean
    of 200 back to back, and from a CUDA-graph replay)."""
    out = {}
    burst, sust, hbm = (float(peaks["bf16_tflops"]), float(peaks["bf16_tflops_sustained"]),
                        float(peaks["hbm_gbs"]))
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    with ClockSampler(local) as clk:
        for name, w in WORKLOADS.items():
            q, k, v = make_inputs(w, device=dev, seed=w.seed)
            rope = lcx.RopeParams(w.mode, w.D, w.base, w.scale, w.original_max_pos, w.alpha,
                                  w.beta, w.pairing)
            o = torch.empty_like(q)
            parts = 3 if (w.split_qk and k.dtype == torch.bfloat16) else 1
            k_rot = torch.empty((parts,) + tuple(k.shape), dtype=k.dtype, device=dev)
            kw = dict(causal=w.causal, window=w.window, sinks=w.sinks,
                      softmax_scale=w.softmax_scale, split_qk=w.split_qk, out=o,
                      status=status, k_rot=k_rot)
            in_bytes = sum(t.numel() * t.element_size() for t in (q, k, v))
            fl = flush if in_bytes < L2_BYTES else None
            tiny = w.L * w.B * w.Hq <= 4096
            n = 200 if tiny else reps
            ms = _call_ms(lambda: lcx.attn_fwd(q, k, v, rope, **kw), stream, n,
                          flush=None if tiny else fl, per_call=not tiny)
            flops = attn_flops(w)
            tf = flops / (ms * 1e-3) / 1e12
            qr, kr = torch.empty_like(q), torch.empty_like(k)

            def rope_qk():
                lcx.apply_rope(q, rope, out=qr)
                lcx.apply_rope(k, rope, out=kr)
            rope_ms = _call_ms(rope_qk, stream, max(reps, 5), flush=fl, per_call=True)
            k_pass_ms = _call_ms(lambda: lcx.apply_rope(k, rope, out=kr), stream,
                                 max(reps, 5), flush=fl, per_call=True)
            rb = rope_bytes(w)
            e = {
                "what": w.description, "ms_per_call": round(ms, 4), "calls": n,
                "timing": ("mean of %d back to back" % n) if tiny else (
                    "median of %d calls, each timed alone" % n),
                "attn_tflops": round(tf, 2), "frac_sustained": round(tf / sust, 4),
                "frac_burst": round(tf / burst, 4),
                "apply_rope_gbs": round(rb / (rope_ms * 1e-3) / 1e9, 1),
                "apply_rope_frac_hbm": round(rb / (rope_ms * 1e-3) / 1e9 / hbm, 4),
                "apply_rope_ms": round(rope_ms, 4),
                "l2": "flushed between calls" if fl is not None else (
                    "inputs larger than L2" if not tiny else "launch-bound latency, L2 warm"),
                "qk_mode": ("split: fp16 q'k' + e5m2 cross terms, fp16 P and V" if w.split_qk
                            else "tf32" if w.dtype == "f32" and w.D == 64 else "bf16"),
                "dtype": w.dtype, "flops_per_call": flops,
            }
            if not w.split_qk:
                # the attention kernel alone: the call minus the keys' rotate pass
                kern = ms - k_pass_ms
                e["kernel_ms"] = round(kern, 4)
                e["kernel_tflops"] = round(flops / (kern * 1e-3) / 1e12, 2)
            if tiny:
                e["latency_us"] = round(ms * 1e3, 2)
                # back-to-back calls from Python are bound by the host's issue
                # time; replayed from a CUDA graph they show the device's own
                g_us, h_us = _graph_and_host_us(lambda: lcx.attn_fwd(q, k, v, rope, **kw))
                e["latency_graph_us"] = round(g_us, 2)
                e["host_issue_us"] = round(h_us, 2)
            assert int(status.item()) == 0, "device watchdog fired in %s" % name
            out[name] = e
            del q, k, v, o, k_rot, qr, kr
            torch.cuda.empty_cache()
    del flush
    torch.cuda.empty_cache()
    out["clocks"] = clk.summary()
    out["peaks"] = {"bf16_tflops": burst, "bf16_tflops_sustained": sust, "hbm_gbs": hbm}
    return out


def oracle_estimates(configs, budget_s=1.5):
    """The oracle beside each workload: the tiny workload timed over its whole
    tensor; for the others a short sample (the heaviest rows of one kv head)
    gives the oracle's FLOP rate, and the full-size CPU time is extrapolated
    from it (labelled an estimate)."""
    import oracle
    for name, e in configs.items():
        w = WORKLOADS.get(name)
        if w is None:
            continue
        if w.L * w.B * w.Hq <= 4096:
            q, k, v = make_inputs(w, device="cpu", seed=w.seed)
            table, ms, _ = oracle.rope_table(w.mode, w.D, w.base, w.scale, w.original_max_pos,
                                             w.alpha, w.beta)
            scale = w.softmax_scale if w.softmax_scale > 0 else None
            t0 = time.perf_counter()
            oracle.attn_full(q.float().numpy(), k.float().numpy(), v.float().numpy(), table, ms,
                             w.pairing, 0, w.causal, w.window, w.sinks, scale)
            secs = time.perf_counter() - t0
            e["oracle_full_s"] = round(secs, 4)
            e["oracle_full_threads"] = oracle.num_threads(0)
            continue
        rate, secs, cores, desc = oracle_sample(w, budget_s=budget_s)
        e["oracle_tflops_sample"] = rate
        e["oracle_full_s_estimate"] = round(attn_flops(w) / (rate * 1e12), 1)
        e["oracle_estimate_from"] = "%s (%.1f s, %d threads); extrapolated, not run" % (
            desc, secs, cores)


def bench_decode(lcx, w, q, k, v, rope, stream, status, reps=20):
    """Decode step on the workload's cache: the last query position of every
    head (q_offset = L - 1) against all L keys, through lcx_attn_fwd_split for a
    few split counts.  HBM-bound: the algorithmic bytes are K and V read once
    (plus q and o); reported against the measured copy bandwidth."""
    if not w.causal or w.L < 2 * 128:
        return None
    qd = q[:, :, -1:].contiguous()
    od = torch.empty_like(qd)
    kw = dict(causal=True, window=w.window, sinks=w.sinks, softmax_scale=w.softmax_scale,
              split_qk=w.split_qk, out=od, status=status, q_offset=w.L - 1)
    # algorithmic bytes: q and o, and the K and V rows of the keys the new token
    # sees (the whole cache, or its window and sinks)
    n_vis = _row_visible(w, w.L - 1)
    kv_row = (k.shape[3] * k.element_size() + v.shape[3] * v.element_size()) * w.B * w.Hkv
    nbytes = n_vis * kv_row + sum(t.numel() * t.element_size() for t in (qd, od))
    sweep = {}
    # the powers of two, and the count that gives every SM one CTA of a kv group
    sms = torch.cuda.get_device_properties(q.device).multi_processor_count
    fill = max(1, min(256, sms // (w.B * w.Hkv)))
    for splits in sorted({1, 8, 16, 32, 64, fill}):
        ws = torch.empty(max(1, lcx.split_workspace_bytes(w.B, w.Hq, 1, w.D, splits)),
                         dtype=torch.uint8, device=q.device)
        for _ in range(3):
            lcx.attn_fwd(qd, k, v, rope, num_splits=splits, workspace=ws, **kw)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            lcx.attn_fwd(qd, k, v, rope, num_splits=splits, workspace=ws, **kw)
        b.record(stream)
        torch.cuda.synchronize()
        sweep[splits] = a.elapsed_time(b) / reps
    best = min(sweep, key=sweep.get)
    # the same step on a cache of keys rotated beforehand (LCX_ATTN_PREROTATED_K)
    k_rot = lcx.apply_rope(k, rope)
    ws = torch.empty(max(1, lcx.split_workspace_bytes(w.B, w.Hq, 1, w.D, best)),
                     dtype=torch.uint8, device=q.device)
    for _ in range(3):
        lcx.attn_fwd(qd, k_rot, v, rope, num_splits=best, workspace=ws, k_prerotated=True, **kw)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(reps):
        lcx.attn_fwd(qd, k_rot, v, rope, num_splits=best, workspace=ws, k_prerotated=True, **kw)
    b.record(stream)
    torch.cuda.synchronize()
    us_rot = a.elapsed_time(b) / reps * 1e3
    del k_rot
    assert int(status.item()) == 0, "device watchdog fired in decode"
    us = sweep[best] * 1e3
    return {"what": "1 new token per head (B=%d, Hq=%d) against %d cached keys (%d of them "
                    "visible), q_offset = L - 1, keys rotated on chip" % (w.B, w.Hq, w.L, n_vis),
            "bound": "hbm", "num_splits": best, "us_per_call": round(us, 2),
            "us_by_splits": {str(s_): round(t * 1e3, 2) for s_, t in sweep.items()},
            "bytes": nbytes, "achieved": round(nbytes / (us * 1e-6) / 1e9, 1), "unit": "GB/s",
            "us_per_call_prerotated_keys": round(us_rot, 2),
            "achieved_prerotated_keys": round(nbytes / (us_rot * 1e-6) / 1e9, 1),
            "launches": (1 if best == 1 else 2) * reps * 2}


def bench_mla(lcx, dev, stream, status, reps=5):
    """Decoupled-RoPE prefill in DeepSeek-V2's head shape (q/k 128 + 64 rotary
    dims with one shared rotary key, v 128): B 1, 16 heads, L 16384, YaRN s=16
    from 4096, causal.  Algorithmic FLOPs: 2 (192 + 128) per visible pair and
    head."""
    B, H, L, Dc, Dr, Dv = 1, 16, 16384, 128, 64, 128
    g = torch.Generator(device=dev).manual_seed(0)
    q = torch.randn((B, H, L, Dc + Dr), generator=g, device=dev).bfloat16()
    kc = torch.randn((B, H, L, Dc), generator=g, device=dev).bfloat16()
    kr = torch.randn((B, 1, L, Dr), generator=g, device=dev).bfloat16()
    v = torch.randn((B, H, L, Dv), generator=g, device=dev).bfloat16()
    o = torch.empty((B, H, L, Dv), dtype=torch.bfloat16, device=dev)
    rope = lcx.RopeParams("yarn", Dr, scale=16.0, original_max_pos=4096)
    k_rot = torch.empty_like(kr)

    def timed(**extra):
        kw = dict(out=o, status=status, k_rope=kr, **extra)
        for _ in range(2):
            lcx.attn_fwd(q, kc, v, rope, **kw)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            lcx.attn_fwd(q, kc, v, rope, **kw)
        b.record(stream)
        torch.cuda.synchronize()
        assert int(status.item()) == 0, "device watchdog fired in the decoupled-RoPE run"
        return a.elapsed_time(b) / reps

    # the shared rotary key rotated once per call (the rotate pass, then the
    # kernel), as in the headline step; and rotated on chip per key tile
    ms = timed(k_rot=k_rot)
    ms_chip = timed()
    flops = 2 * (Dc + Dr + Dv) * visible_pairs(L) * B * H
    return {"what": "decoupled RoPE prefill, B 1, 16 heads, L 16384, q/k 128+64 (shared rotary "
                    "key rotated once per call), v 128, YaRN s=16", "ms_per_call": round(ms, 3),
            "achieved": round(flops / (ms * 1e-3) / 1e12, 1), "unit": "TFLOP/s",
            "achieved_key_rotated_on_chip": round(flops / (ms_chip * 1e-3) / 1e12, 1),
            "launches": 2 * reps + reps}


def bench_reference(args, world, rank):
    """The reference arm: the fp64 oracle as it stands, on host cores."""
    if rank != 0:
        return None
    w = WORKLOADS[args.workload]
    vals, secs_all = [], 0.0
    for s in range(args.warmup + args.steps):
        val, secs, cores, desc = oracle_sample(w, budget_s=args.cpu_budget / max(1, args.steps),
                                               seed=s)
        if s >= args.warmup:
            vals.append(val)
            secs_all += secs
    value = statistics.mean(vals)
    return {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(secs_all / args.steps * 1e3, 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
        "impl": "reference",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "L": w.L, "D": w.D,
                   "rope": w.mode},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def relaunch(n):
    """Run this script as n ranks under torchrun (one per GPU, rendezvous on
    127.0.0.1) with the same arguments; returns torchrun's exit status.  Rank 0
    prints the JSON line."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           "--nproc-per-node", str(n), "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=HEADLINE, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="lcx", choices=["lcx", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--cpu-budget-per-config", type=float, default=1.5)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-workload measurements (the configs object)")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip decode, decoupled-RoPE and per-workload measurements")
    ap.add_argument("--batch", type=int, default=0,
                    help="override the workload's batch size (smaller captures for profiling; "
                         "the line's config records it)")
    ap.add_argument("--shard", default="replicas", choices=["replicas", "heads"],
                    help="N > 1: independent replicas (weak scaling) or one batch split by "
                         "kv heads (strong scaling)")
    ap.add_argument("--decode-only", action="store_true",
                    help="only the split-KV decode measurement on the workload's cache "
                         "(prints its object; for profiling, not a bench line)")
    args = ap.parse_args()
    env_world = os.environ.get("WORLD_SIZE")
    if env_world is None and args.gpus > 1:
        # not launched under torchrun: start the N ranks here
        sys.exit(relaunch(args.gpus))
    if env_world is not None and int(env_world) != args.gpus:
        print("bench.py: --gpus %d but WORLD_SIZE=%s; launch one rank per GPU with "
              "--gpus equal to the number of ranks" % (args.gpus, env_world), file=sys.stderr)
        sys.exit(2)
    if args.decode_only:
        import ntk_rope_flashattn_b200 as lcx
        w = WORKLOADS[args.workload]
        dev = torch.device("cuda", 0)
        q, k, v = make_inputs(w, device=dev, seed=rank_seed(w, 0))
        rope = lcx.RopeParams(w.mode, w.D, w.base, w.scale, w.original_max_pos, w.alpha,
                              w.beta, w.pairing)
        status = torch.zeros(1, dtype=torch.int32, device=dev)
        res = bench_decode(lcx, w, q, k, v, rope, torch.cuda.current_stream(dev), status,
                           reps=args.steps)
        print(json.dumps(res), flush=True)
        return
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        res = bench_reference(args, world, rank)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    world, rank, local = dist_setup(args)
    try:
        res = bench_gpu(args, world, rank, local)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
