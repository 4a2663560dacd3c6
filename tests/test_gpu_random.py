"""Seeded random combinations of the attention call's options against the fp64
oracle ("Long Context: RoPE / YaRN / NTK / MLA", 2.4 rope_attention; "8.3
长上下文技术", 8.3.4): head dim, operand type, RoPE mode and pairing, GQA group
(odd ones included), batch, ragged lengths, causal or not, sliding window and
sinks, split QK^T, keys rotated once into a buffer, a chunk of queries at a
position offset (down to a single decode row), and split-KV.

The hand-written cases elsewhere pin each option; this sweep checks that they
compose.  Every draw is fixed by its index, so a failure names a reproducible
configuration.  Tolerances are the prefill tests' (test_gpu_attn.py).
"""
import numpy as np
import pytest
import torch

import ntk_rope_flashattn_b200 as lcx
from test_gpu_attn import compare
from test_gpu_decode import oracle_rows
from workloads import Workload, make_inputs

pytestmark = pytest.mark.gpu

N_DRAWS = 120


def draw(i):
    """Configuration i: (workload, call options, query rows of the call)."""
    r = np.random.default_rng(7919 + i)
    D = int(r.choice([64, 128]))
    dtype = "f32" if r.random() < 0.15 else "bf16"
    G = int(r.choice([1, 2, 3, 4, 8]))
    Hkv = int(r.choice([1, 2]))
    B = int(r.choice([1, 2]))
    Lk = int(r.integers(1, 900))
    mode = str(r.choice(["plain", "pi", "ntk", "yarn"]))
    pairing = str(r.choice(["half", "interleaved"]))
    causal = bool(r.random() < 0.85)
    window = int(r.integers(1, Lk + 1)) if causal and r.random() < 0.4 else 0
    sinks = int(r.integers(0, 140)) if window and r.random() < 0.5 else 0
    w = Workload("draw%d" % i, B=B, Hq=G * Hkv, Hkv=Hkv, L=Lk, D=D, dtype=dtype, mode=mode,
                 scale=float(r.choice([2.0, 4.0, 8.0])), original_max_pos=128,
                 pairing=pairing, causal=causal, window=window, sinks=sinks,
                 seed=int(r.integers(0, 1000)))
    # all rows (prefill), or the last Lq rows at positions Lk - Lq .. Lk - 1: a
    # chunk, or 1-3 rows (decode)
    if not causal or r.random() < 0.5:
        Lq = Lk
    elif r.random() < 0.35:
        Lq = min(Lk, int(r.integers(1, 4)))
    else:
        Lq = int(r.integers(1, Lk + 1))
    opts = dict(split_qk=bool(r.random() < 0.25), rotate_k_once=bool(r.random() < 0.4),
                num_splits=int(r.choice([1, 1, 2, 5])))
    return w, opts, Lq


@pytest.mark.parametrize("i", range(N_DRAWS))
def test_random_configuration(i):
    w, opts, Lq = draw(i)
    q_all, k, v = make_inputs(w, device="cuda")
    q = q_all[:, :, w.L - Lq:]
    rope = lcx.RopeParams(w.mode, w.D, w.base, w.scale, w.original_max_pos, w.alpha, w.beta,
                          w.pairing)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = lcx.attn_fwd(q, k, v, rope, causal=w.causal, window=w.window, sinks=w.sinks,
                          q_offset=w.L - Lq, return_lse=True, status=status, **opts)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, (w, opts, Lq)
    ref_o, ref_lse = oracle_rows(q, k, v, rope, w.L - Lq, w.causal, w.window, w.sinks)
    compare(o.float().cpu().numpy(), lse.cpu().numpy(), ref_o, ref_lse,
            24 if w.dtype == "f32" else 8)


N_DRAWS_MLA = 40


def draw_mla(i):
    """Decoupled-RoPE configuration i: q/k head dim d_C + d_R with d_R = 64 (d_C
    128 or 64), value dim 128, the rotary key shared by every head."""
    r = np.random.default_rng(104729 + i)
    Dc = int(r.choice([128, 64]))
    G = int(r.choice([1, 2, 3, 4]))
    Hkv = int(r.choice([1, 2]))
    Lk = int(r.integers(1, 700))
    window = int(r.integers(1, Lk + 1)) if r.random() < 0.35 else 0
    sinks = int(r.integers(0, 100)) if window and r.random() < 0.5 else 0
    Lq = Lk if r.random() < 0.5 else int(r.integers(1, Lk + 1))
    rope = dict(mode=str(r.choice(["plain", "pi", "ntk", "yarn"])),
                scale=float(r.choice([2.0, 4.0, 8.0])), original_max_pos=128,
                pairing=str(r.choice(["half", "interleaved"])))
    opts = dict(rotate_k_once=bool(r.random() < 0.5), num_splits=int(r.choice([1, 1, 3])))
    return dict(B=int(r.choice([1, 2])), Hq=G * Hkv, Hkv=Hkv, Lk=Lk, Lq=Lq, Dc=Dc,
                window=window, sinks=sinks, seed=int(r.integers(0, 1000)), rope=rope,
                opts=opts)


@pytest.mark.parametrize("i", range(N_DRAWS_MLA))
def test_random_decoupled_rope(i):
    from test_gpu_mla import mla_inputs, oracle_mla
    c = draw_mla(i)
    Dr, Dv = 64, 128
    q_all, kc, kr, v = mla_inputs(c["B"], c["Hq"], c["Hkv"], c["Lk"], c["Dc"], Dr, Dv,
                                  seed=c["seed"])
    q = q_all[:, :, c["Lk"] - c["Lq"]:]
    rope = lcx.RopeParams(head_dim=Dr, **c["rope"])
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = lcx.attn_fwd(q, kc, v, rope, k_rope=kr, window=c["window"], sinks=c["sinks"],
                          q_offset=c["Lk"] - c["Lq"], return_lse=True, status=status,
                          **c["opts"])
    torch.cuda.synchronize()
    assert int(status.item()) == 0, c
    ref = oracle_mla(q, kc, kr, v, rope, c["Lk"] - c["Lq"], c["window"], c["sinks"])
    compare(o.float().cpu().numpy(), lse.cpu().numpy(), ref[0], ref[1])
