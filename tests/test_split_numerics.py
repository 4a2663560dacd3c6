"""Why the split-QK^T mode forms its logits the way it does (a CPU model).

The outlier workload ("Long Context: RoPE / YaRN / NTK / MLA", 10.1-10.2
sliding window and sinks, 6.2-6.4 YaRN s = 8; Q, K, V ~ N(0, 1) with 1% of the
entries x8) produces logits large enough that rounding the rotated operands
q', k' to bf16 alone moves the output far beyond the 2e-2 bound.  This test
models, in float64 torch on the CPU, only the operand roundings of candidate
ways to form QK^T (everything else exact, P rounded to bf16, o to bf16) and
compares them with the fp64 definition on seeded 128-row blocks shaped like the
workload (window 4096 + 4 sinks):

  bf16          one bf16 product                       (the plain mode)
  f16           one fp16 product
  bf16x3        bf16 hi/lo parts, hi.hi + hi.lo + lo.hi (three products)
  f16_x8        fp16 part h and residual r = x' - h:
                qh.kh + [e5m2(qh) | e5m2(qr)].[e5m2(kr) | e5m2(kh)]  (the kernel's)

with P rounded to bf16 for PV, and for the kernel's split mode also with P
(and V, exactly) in fp16 (f16_x8_pf16).  The kernel's logits (f16_x8) must
meet the bound the way three bf16 products do (what is left is mostly the
bf16 rounding of P, common to both), and bf16 alone must not; a single fp16
product is measurably worse than either; and fp16 weights must not add
error.  The CUDA path is not involved; its own parity
against the oracle is in the GPU tests.
"""
import math

import numpy as np
import pytest
import torch

import oracle

D, L, W, S = 128, 65536, 4096, 4
BOUND = 2e-2


def _gen(shape, g):
    x = torch.randn(shape, generator=g, dtype=torch.float32)
    m = torch.rand(shape, generator=g, dtype=torch.float32) < 0.01
    x[m] *= 8
    return x.bfloat16().double()


def _rot(x, pos, theta, scale):
    ang = pos[:, None].double() * theta[None, :]
    c, s = torch.cos(ang), torch.sin(ang)
    a, b = x[:, :D // 2], x[:, D // 2:]
    return torch.cat([a * c - b * s, a * s + b * c], 1) * scale


def _r(x, dt):
    return x.float().to(dt).double()


def _scores(kind, q, k):
    if kind == "exact":
        return q @ k.T
    if kind == "bf16":
        return _r(q, torch.bfloat16) @ _r(k, torch.bfloat16).T
    if kind == "f16":
        return _r(q, torch.float16) @ _r(k, torch.float16).T
    if kind == "bf16x3":
        qh, kh = _r(q, torch.bfloat16), _r(k, torch.bfloat16)
        ql, kl = _r(q - qh, torch.bfloat16), _r(k - kh, torch.bfloat16)
        return qh @ kh.T + qh @ kl.T + ql @ kh.T
    if kind == "f16_x8":
        qh, kh = _r(q, torch.float16), _r(k, torch.float16)
        e5 = torch.float8_e5m2
        q8 = torch.cat([_r(qh, e5), _r(q - qh, e5)], 1)
        k8 = torch.cat([_r(k - kh, e5), _r(kh, e5)], 1)
        return qh @ kh.T + q8 @ k8.T
    raise ValueError(kind)


def _attend(s, mask, v, p_type):
    x = s.masked_fill(~mask, -math.inf)
    p = torch.exp(x - x.max(1, keepdim=True).values)
    if p_type is not None:
        p = _r(p, p_type)
    return (p @ v) / p.sum(1, keepdim=True)


def _excess(o, ref):
    """|o - ref| beyond half a bf16 ulp of |ref| where |ref| >= 4 (the GPU tests'
    comparison), raw below."""
    ob = _r(o, torch.bfloat16)
    err = (ob - ref).abs()
    a = ref.abs().clamp_min(1e-30)
    half_ulp = torch.pow(2.0, torch.floor(torch.log2(a)) - 8)
    return torch.where(ref.abs() >= 4, err - half_ulp, err).max().item(), err.mean().item()


def test_split_operands_meet_the_bound_where_bf16_does_not():
    table, ms, _ = oracle.rope_table("yarn", D, 10000.0, 8.0, 8192, 1.0, 32.0)
    theta = torch.tensor(np.asarray(table, dtype=np.float64))
    ms = float(ms)
    scale = ms / math.sqrt(D)   # logit scale on (q' without mscale) . (k' with it)
    g = torch.Generator().manual_seed(2024)
    worst = {k: 0.0 for k in ("bf16", "f16", "bf16x3", "f16_x8", "f16_x8_pf16")}
    means = {k: [] for k in worst}
    for _ in range(6):
        k = _gen((L, D), g)
        v = _gen((L, D), g)
        q0 = int(torch.randint(W // 128, L // 128, (1,), generator=g)) * 128
        kidx = torch.cat([torch.arange(0, S), torch.arange(q0 - W + 1, q0 + 128)])
        kr = _rot(k[kidx], kidx, theta, ms)
        vv = v[kidx]
        qpos = torch.arange(q0, q0 + 128)
        mask = (kidx[None] <= qpos[:, None]) & ((qpos[:, None] - kidx[None] < W) |
                                                 (kidx[None] < S))
        for _h in range(4):
            qr = _rot(_gen((128, D), g), qpos, theta, 1.0)
            ref = _attend(_scores("exact", qr, kr) * scale, mask, vv, None)
            for kind in worst:
                # P rounded to bf16 for PV (plain mode), the kernel's split mode
                # rounds P (and its bf16 V, exactly) to fp16
                pt = torch.float16 if kind == "f16_x8_pf16" else torch.bfloat16
                sk = "f16_x8" if kind == "f16_x8_pf16" else kind
                e, m = _excess(_attend(_scores(sk, qr, kr) * scale, mask, vv, pt), ref)
                worst[kind] = max(worst[kind], e)
                means[kind].append(m)
    print({k: round(v_, 4) for k, v_ in worst.items()})
    assert worst["bf16"] > BOUND                       # why the split mode exists
    assert worst["f16_x8"] <= BOUND                    # the split mode's logits
    assert worst["f16_x8"] <= worst["bf16x3"] + 2e-3   # as good as three bf16 products
    assert worst["f16"] > worst["f16_x8"] + 2e-3       # the cross terms are needed
    # with P in fp16 P's share of the remaining error goes (what is left is
    # mostly the output's own bf16 rounding, up to 2^-7 just below |o| = 4)
    assert worst["f16_x8_pf16"] <= worst["f16_x8"]
    assert np.mean(means["f16_x8_pf16"]) <= 2e-3
