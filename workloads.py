"""Seeded synthetic workloads: shapes, RoPE settings and input tensors.

This module holds the workload descriptions and the seeded input generators
shared by the CUDA path's tests/benchmark and by the CPU oracle's tests.  It
holds none of the method's arithmetic (no frequencies, rotations or softmax):
only sizes, settings and random draws.

Input recipe (one fresh generator per workload, seed 0):
  Q, K, V ~ N(0, 1) drawn in fp32 in that order; for the outlier workload three
  Bernoulli(0.01) masks (for Q, K, V, in that order) drawn afterwards from the
  same generator multiply the selected entries by 8; then the tensors are cast
  (round-to-nearest-even) to the workload's dtype.
"""
from dataclasses import dataclass, asdict

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    L: int
    D: int
    dtype: str                 # "bf16" or "f32"
    mode: str                  # "none" | "plain" | "pi" | "ntk" | "yarn"
    base: float = 10000.0
    scale: float = 1.0         # s = L_new / L_train
    original_max_pos: int = 4096
    alpha: float = 1.0
    beta: float = 32.0
    pairing: str = "half"
    causal: bool = True
    window: int = 0
    sinks: int = 0
    softmax_scale: float = 0.0  # 0 -> 1/sqrt(D)
    outlier_frac: float = 0.0
    outlier_mult: float = 8.0
    split_qk: bool = False     # form QK^T from fp16 + e5m2 cross parts (outlier-heavy inputs)
    seed: int = 0
    description: str = ""

    def rope(self):
        return dict(mode=self.mode, head_dim=self.D, base=self.base, scale=self.scale,
                    original_max_pos=self.original_max_pos, alpha=self.alpha,
                    beta=self.beta, pairing=self.pairing)

    def with_(self, **kw):
        d = asdict(self)
        d.update(kw)
        return Workload(**d)

    @property
    def torch_dtype(self):
        return {"bf16": torch.bfloat16, "f32": torch.float32}[self.dtype]


# The five workloads the pages' long-context settings call for.
WORKLOADS = {
    "tiny_L256_D64": Workload(
        "tiny_L256_D64", B=1, Hq=1, Hkv=1, L=256, D=64, dtype="f32", mode="plain",
        softmax_scale=1.0 / 8.0,
        description="batch 1, 1 head, seq 256, head_dim 64, fp32, plain RoPE base 1e4, causal"),
    "llama3_8b_L8192": Workload(
        "llama3_8b_L8192", B=1, Hq=32, Hkv=8, L=8192, D=128, dtype="bf16", mode="plain",
        description="Llama-3-8B-shaped layer: 32 Q / 8 KV heads, head_dim 128, seq 8192, plain RoPE"),
    "pi_L32768_s4": Workload(
        "pi_L32768_s4", B=1, Hq=32, Hkv=8, L=32768, D=128, dtype="bf16", mode="pi",
        scale=4.0, original_max_pos=8192,
        description="PI: L_train 8192 -> seq 32768 (s=4), 32/8 heads, head_dim 128"),
    "ntk_L32768_s4": Workload(
        "ntk_L32768_s4", B=1, Hq=32, Hkv=8, L=32768, D=128, dtype="bf16", mode="ntk",
        scale=4.0, original_max_pos=8192,
        description="NTK-aware base 1e4*4^(128/126): seq 32768, 32/8 heads, head_dim 128"),
    "yarn_L131072_s16": Workload(
        "yarn_L131072_s16", B=1, Hq=32, Hkv=8, L=131072, D=128, dtype="bf16", mode="yarn",
        scale=16.0, original_max_pos=8192, alpha=1.0, beta=32.0,
        description="YaRN 8K->128K: seq 131072, s=16, alpha 1, beta 32, 32/8 heads, head_dim 128"),
    "sink_window_L65536": Workload(
        "sink_window_L65536", B=4, Hq=32, Hkv=8, L=65536, D=128, dtype="bf16", mode="yarn",
        scale=8.0, original_max_pos=8192, alpha=1.0, beta=32.0, window=4096, sinks=4,
        outlier_frac=0.01, outlier_mult=8.0, split_qk=True,
        description="4 sink tokens + window 4096, batch 4, seq 65536, YaRN s=8, 1% outliers x8"),
}

# The workload the headline metric (fused YaRN-RoPE causal attention prefill) is quoted on.
HEADLINE = "yarn_L131072_s16"


def make_inputs(w: Workload, device="cpu", seed=None):
    """Seeded Q [B,Hq,L,D], K [B,Hkv,L,D], V [B,Hkv,L,D] in the workload's dtype."""
    g = torch.Generator(device=device)
    g.manual_seed(w.seed if seed is None else seed)
    shp_q = (w.B, w.Hq, w.L, w.D)
    shp_kv = (w.B, w.Hkv, w.L, w.D)
    q = torch.randn(shp_q, generator=g, dtype=torch.float32, device=device)
    k = torch.randn(shp_kv, generator=g, dtype=torch.float32, device=device)
    v = torch.randn(shp_kv, generator=g, dtype=torch.float32, device=device)
    if w.outlier_frac > 0:
        for t in (q, k, v):
            m = torch.rand(t.shape, generator=g, dtype=torch.float32, device=device) < w.outlier_frac
            t[m] *= w.outlier_mult
            del m
    dt = w.torch_dtype
    return q.to(dt), k.to(dt), v.to(dt)


def sample_rows(w: Workload, n_random=32, seed=1, batches=None):
    """Query indices to check at full size: boundary rows plus seeded random rows."""
    L = w.L
    fixed = {0, 1, 127, 128, 129, L // 2, L - 1, L - 2}
    if w.window:
        fixed |= {w.window - 1, w.window, w.window + w.sinks}
    rows = sorted(i for i in fixed if 0 <= i < L)
    g = torch.Generator().manual_seed(seed)
    rnd = torch.randint(0, L, (n_random,), generator=g).tolist()
    rows = sorted(set(rows) | set(rnd))
    if batches is None:
        batches = sorted({0, w.B - 1})
    return rows, batches


def visible_pairs(L, causal=True, window=0, sinks=0):
    """Exact count of visible (query, key) pairs of one (batch, head): the
    causal-adjusted work unit the attention FLOP count is based on."""
    if not causal:
        return L * L
    if window <= 0 or window >= L:
        return L * (L + 1) // 2
    total = 0
    # rows i < window see keys 0..i (i+1 keys)
    n1 = min(window, L)
    total += n1 * (n1 + 1) // 2
    # rows i >= window see the window (W keys) plus sinks j < min(S, i-W+1)
    for_rows = L - n1
    total += for_rows * window
    S = sinks
    if S > 0:
        # extra sink keys for row i: number of j < S with j <= i - W, i.e. min(S, i-W+1)
        # summed over i in [W, L): rows with i - W + 1 >= S contribute S
        i0 = window  # first row beyond the window
        # rows i in [W, W+S-1) contribute i-W+1 (1..S-1)
        k = min(S - 1, L - i0)
        total += k * (k + 1) // 2
        rest = L - i0 - k
        if rest > 0:
            total += rest * S
    return total


def attn_flops(w: Workload):
    """Algorithmic attention FLOPs: 4 * D per visible pair (QK^T and PV), per (b, hq)."""
    return 4 * w.D * visible_pairs(w.L, w.causal, w.window, w.sinks) * w.B * w.Hq


def rope_bytes(w: Workload):
    """Bytes one out-of-place RoPE pass over Q and K moves (read + write)."""
    es = 2 if w.dtype == "bf16" else 4
    return 2 * es * w.B * (w.Hq + w.Hkv) * w.L * w.D
