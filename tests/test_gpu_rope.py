"""GPU parity of lcx_apply_rope against the fp64 oracle.

Tolerance (derived from the arithmetic): the kernel forms the angle exactly in
fp64, reduces it to [-pi, pi], evaluates cos/sin in fp32 (error below 2^-21) and
rotates with two fp32 products, so its fp32 pre-rounding value y~ satisfies
|y~ - y| <= delta = 2^-19 * ms * (|x_p| + |x_q|).  The stored value is y~ rounded
once to the output type, so |y_gpu - y| <= delta + ulp(|y| + delta) / 2.
"""
import numpy as np
import pytest
import torch

import ntk_rope_flashattn_b200 as lcx
import oracle
from workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


def ulp(a, dtype):
    a = np.maximum(np.abs(a), np.finfo(np.float32).tiny)
    mant = 7 if dtype == torch.bfloat16 else 23
    return np.exp2(np.floor(np.log2(a)) - mant)


def check_rotation(x, y, rope, pos_offset=0):
    """Compare y (device) with the oracle rotation of x (device), row by row."""
    B, H, L, D = x.shape
    table, ms, flags = oracle.rope_table(rope.mode, D, rope.base, rope.scale,
                                         rope.original_max_pos, rope.alpha, rope.beta)
    xs = x.float().cpu().numpy().reshape(-1, D)
    pos = np.tile(np.arange(L) + pos_offset, B * H)
    ref = oracle.rotate_rows(xs, pos, table, ms, rope.pairing)
    got = y.float().cpu().numpy().reshape(-1, D).astype(np.float64)
    half = D // 2
    if rope.pairing == "half":
        partner = np.concatenate([np.arange(half, D), np.arange(half)])
    else:
        partner = np.arange(D) ^ 1
    delta = 2.0 ** -19 * float(ms) * (np.abs(xs) + np.abs(xs[:, partner]))
    tol = delta + 0.5 * ulp(np.abs(ref) + delta, x.dtype)
    err = np.abs(got - ref)
    bad = err > tol
    assert not bad.any(), "max err/tol %.3g at %s" % ((err / tol).max(), np.argwhere(bad)[:5])


CASES = [
    # (B, H, L, D, dtype, mode, scale, pairing, pos_offset)
    (1, 4, 1, 128, torch.bfloat16, "plain", 1.0, "half", 0),
    (2, 3, 129, 128, torch.bfloat16, "yarn", 16.0, "half", 0),
    (1, 8, 300, 64, torch.bfloat16, "ntk", 4.0, "half", 7),
    (1, 2, 257, 128, torch.bfloat16, "pi", 4.0, "interleaved", 0),
    (1, 2, 100, 64, torch.float32, "plain", 1.0, "half", 0),
    (1, 2, 100, 64, torch.float32, "yarn", 8.0, "interleaved", 131000),
    (1, 1, 64, 256, torch.bfloat16, "yarn", 4.0, "half", 0),
    (1, 2, 33, 96, torch.bfloat16, "plain", 1.0, "half", 0),
]


@pytest.mark.parametrize("B,H,L,D,dt,mode,s,pairing,off", CASES)
def test_apply_rope_matches_oracle(B, H, L, D, dt, mode, s, pairing, off):
    g = torch.Generator(device="cuda").manual_seed(0)
    x = torch.randn((B, H, L, D), generator=g, device="cuda").to(dt)
    rope = lcx.RopeParams(mode, D, scale=s, original_max_pos=2048, pairing=pairing)
    y = lcx.apply_rope(x, rope, pos_offset=off)
    torch.cuda.synchronize()
    check_rotation(x, y, rope, off)


def test_apply_rope_in_place_and_strided():
    """In place equals out of place; a [B, L, H, D] buffer viewed as [B, H, L, D]
    (non-contiguous strides) is handled."""
    g = torch.Generator(device="cuda").manual_seed(1)
    base = torch.randn((2, 200, 4, 128), generator=g, device="cuda").bfloat16()
    x = base.permute(0, 2, 1, 3)                       # [B, H, L, D] view
    rope = lcx.RopeParams("yarn", 128, scale=8.0, original_max_pos=64)
    y = lcx.apply_rope(x, rope)
    torch.cuda.synchronize()
    check_rotation(x, y, rope)
    x2 = x.clone()
    lcx.apply_rope(x2, rope, inplace=True)
    torch.cuda.synchronize()
    assert torch.equal(x2, y)


@pytest.mark.parametrize("name", ["yarn_L131072_s16", "sink_window_L65536"])
def test_apply_rope_full_size_sampled(name):
    """Full-size Q and K of the long workloads; every head at sampled positions."""
    w = WORKLOADS[name]
    q, k, _ = make_inputs(w, device="cuda")
    rope = lcx.RopeParams(w.mode, w.D, w.base, w.scale, w.original_max_pos, w.alpha, w.beta)
    for x in (q, k):
        y = lcx.apply_rope(x, rope)
        torch.cuda.synchronize()
        idx = torch.tensor([0, 1, 4095, 8191, w.L // 2, w.L - 1], device="cuda")
        for b in sorted({0, w.B - 1}):
            xs = x[b:b + 1].index_select(2, idx)
            ys = y[b:b + 1].index_select(2, idx)
            table, ms, _ = oracle.rope_table(w.mode, w.D, w.base, w.scale, w.original_max_pos,
                                             w.alpha, w.beta)
            xr = xs.float().cpu().numpy().reshape(-1, w.D)
            pos = np.tile(idx.cpu().numpy(), xs.shape[1])
            ref = oracle.rotate_rows(xr, pos, table, ms, "half")
            got = ys.float().cpu().numpy().reshape(-1, w.D)
            partner = np.concatenate([np.arange(w.D // 2, w.D), np.arange(w.D // 2)])
            delta = 2.0 ** -19 * float(ms) * (np.abs(xr) + np.abs(xr[:, partner]))
            tol = delta + 0.5 * ulp(np.abs(ref) + delta, torch.bfloat16)
            assert (np.abs(got - ref) <= tol).all()
        del y


def test_apply_rope_dynamic_ntk_uses_offset_plus_length():
    """Dynamic NTK in lcx_apply_rope takes the context length pos_offset + L."""
    g = torch.Generator(device="cuda").manual_seed(3)
    x = torch.randn((1, 2, 100, 128), generator=g, device="cuda").bfloat16()
    rope = lcx.RopeParams("dynamic_ntk", 128, original_max_pos=4096)
    y = lcx.apply_rope(x, rope, pos_offset=30000)
    torch.cuda.synchronize()
    table, ms, _ = oracle.rope_table("dynamic_ntk", 128, original_max_pos=4096, seq_len=30100)
    xs = x.float().cpu().numpy().reshape(-1, 128)
    pos = np.tile(np.arange(100) + 30000, 2)
    ref = oracle.rotate_rows(xs, pos, table, ms, "half")
    partner = np.concatenate([np.arange(64, 128), np.arange(64)])
    delta = 2.0 ** -19 * (np.abs(xs) + np.abs(xs[:, partner]))
    tol = delta + 0.5 * ulp(np.abs(ref) + delta, torch.bfloat16)
    assert (np.abs(y.float().cpu().numpy().reshape(-1, 128) - ref) <= tol).all()
