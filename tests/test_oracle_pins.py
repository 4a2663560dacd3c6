"""Pins for the fp64 CPU oracle: values the pages print or state, closed forms,
invariants and brute force -- never the oracle's own formula retyped.

Each test names the page and section whose statement it checks.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from conftest import load_mask, load_pins
import workloads

PINS = load_pins()


def pin(name, got):
    val, tol, src = PINS[name]
    assert abs(got - val) <= tol, f"{name}: got {got!r}, expected {val} +- {tol} ({src})"


def ntk_base_from_table(theta_fp64, D):
    # theta'_1 = b'^(-2/D)  =>  b' = theta'_1^(-D/2)
    return math.exp(-(D / 2) * math.log(theta_fp64[1]))


# --------------------------------------------------------------------------
# frequency tables
# --------------------------------------------------------------------------

def test_plain_d64_printed_frequencies():
    """"长上下文外推", section 5.3: printed frequencies / degrees / period for d=64."""
    th, ms = oracle.rope_theta_fp64("plain", 64)
    assert ms == 1.0
    pin("d64_freq_0", th[0])
    pin("d64_freq_16", th[16])
    pin("d64_freq_31", th[31])
    pin("d64_deg_0", math.degrees(th[0]))
    pin("d64_deg_16", math.degrees(th[16]))
    pin("d64_deg_31", math.degrees(th[31]))
    pin("d64_period_31", 2 * math.pi / th[31])


def _angle_deg(y):
    return math.degrees(math.atan2(y[1], y[0])) % 360.0


@pytest.mark.parametrize("pairing", ["half", "interleaved"])
def test_slow_pair_angles_train_vs_extrapolated(pairing):
    """"长上下文外推", section 6.3: pair 31 of d=64 reaches 31.3 deg at the last of
    4096 positions and 62.6 deg at the last of 8192 (rotating a unit vector)."""
    D = 64
    table, ms, _ = oracle.rope_table("plain", D)
    x = np.zeros((2, D), dtype=np.float32)
    p, q = (31, 63) if pairing == "half" else (62, 63)
    x[:, p] = 1.0
    y = oracle.rotate_rows(x, np.array([4095, 8191]), table, ms, pairing)
    pin("d64_train_deg", _angle_deg((y[0, p], y[0, q])))
    pin("d64_extrap_deg", _angle_deg((y[1, p], y[1, q])))


@pytest.mark.parametrize("s,name", [(2, "ntk_b1e6_d64_s2"), (4, "ntk_b1e6_d64_s4"),
                                    (8, "ntk_b1e6_d64_s8"), (32, "ntk_b1e6_d64_s32")])
def test_ntk_printed_rope_theta_table(s, name):
    """"长上下文外推", section 15.1: printed NTK rope_theta for base 1e6, head_dim 64."""
    th, _ = oracle.rope_theta_fp64("ntk", 64, base=1e6, scale=s)
    pin(name, ntk_base_from_table(th, 64))


def test_ntk_stated_bases():
    """plumephp NTK comment (1.7e5 for 8K->128K at d=128), doc.minddiy homework 1
    (82,684.6 at s=8, d=128; exponent 1.0159) and section 14 (about 86000 at d=64)."""
    th, _ = oracle.rope_theta_fp64("ntk", 128, base=1e4, scale=16)
    pin("ntk_b1e4_d128_s16", ntk_base_from_table(th, 128))
    th, _ = oracle.rope_theta_fp64("ntk", 128, base=1e4, scale=8)
    b = ntk_base_from_table(th, 128)
    pin("ntk_b1e4_d128_s8", b)
    pin("ntk_exp_d128", math.log(b / 1e4) / math.log(8))
    th, _ = oracle.rope_theta_fp64("ntk", 64, base=1e4, scale=8)
    pin("ntk_b1e4_d64_s8", ntk_base_from_table(th, 64))


@pytest.mark.parametrize("D,s", [(64, 2.0), (128, 4.0), (128, 16.0)])
def test_ntk_end_frequencies(D, s):
    """"Long Context: RoPE / YaRN / NTK / MLA", section 5.2: NTK keeps theta_0 and
    divides the lowest frequency by s; ratio s^(-2i/(D-2)) in between ("8.3", 8.3.2)."""
    plain, _ = oracle.rope_theta_fp64("plain", D)
    ntk, _ = oracle.rope_theta_fp64("ntk", D, scale=s)
    assert ntk[0] == 1.0
    assert math.isclose(ntk[-1], plain[-1] / s, rel_tol=1e-13)
    i = np.arange(D // 2)
    np.testing.assert_allclose(ntk / plain, s ** (-2.0 * i / (D - 2)), rtol=1e-12)


@pytest.mark.parametrize("s", [2.0, 4.0, 8.0, 16.0, 64.0])
def test_pi_divides_every_frequency(s):
    """"Long Context: RoPE / YaRN / NTK / MLA", section 4.2: PI divides every theta
    by s; for s = 2^k the fp32 table is exactly the plain table over s."""
    for D in (64, 128):
        plain, ms0, _ = oracle.rope_table("plain", D)
        pi, ms1, _ = oracle.rope_table("pi", D, scale=s)
        assert ms0 == ms1 == 1.0
        np.testing.assert_array_equal(pi, plain / np.float32(s))


def test_pi_equals_scaled_positions():
    """Section 4.2 (and "8.3" 8.3.2): rotating at m with theta/s equals rotating at
    m/s with theta, for positions divisible by s."""
    D, s = 128, 4
    plain, _, _ = oracle.rope_table("plain", D)
    pi, _, _ = oracle.rope_table("pi", D, scale=s)
    rng = np.random.default_rng(0)
    x = rng.standard_normal((64, D)).astype(np.float32)
    m = rng.integers(0, 30000, 64) * s
    a = oracle.rotate_rows(x, m, pi, 1.0)
    b = oracle.rotate_rows(x, m // s, plain, 1.0)
    np.testing.assert_allclose(a, b, atol=1e-12, rtol=0)


@pytest.mark.parametrize("mode", ["yarn", "ntk", "pi"])
def test_scale_one_is_plain(mode):
    """With s = 1 every extension mode is plain RoPE (no interpolation, mscale 1)."""
    for D in (64, 128):
        plain, _, _ = oracle.rope_table("plain", D)
        t, ms, _ = oracle.rope_table(mode, D, scale=1.0, original_max_pos=8192)
        np.testing.assert_array_equal(t, plain)
        assert ms == 1.0


def test_yarn_ramp_regions():
    """"Long Context: RoPE / YaRN / NTK / MLA", section 6.2 and "8.3" 8.3.3:
    theta' = theta where r >= beta, theta/s where r <= alpha, and in between the
    multiplier (r-alpha)/(beta-alpha)*(1-1/s)+1/s written in 8.3.3's form."""
    D, s, Ltr, a, b = 128, 16.0, 8192, 1.0, 32.0
    plain, _ = oracle.rope_theta_fp64("plain", D)
    yarn, ms = oracle.rope_theta_fp64("yarn", D, scale=s, original_max_pos=Ltr, alpha=a, beta=b)
    r = Ltr / (2 * math.pi / plain)        # turns within the training length
    gamma = yarn / plain
    hi, lo = r >= b, r <= a
    assert hi.sum() > 0 and lo.sum() > 0
    np.testing.assert_allclose(gamma[hi], 1.0, rtol=1e-14)
    np.testing.assert_allclose(gamma[lo], 1.0 / s, rtol=1e-14)
    mid = ~(hi | lo)
    expect = (r[mid] - a) / (b - a) * (1 - 1 / s) + 1 / s
    np.testing.assert_allclose(gamma[mid], expect, rtol=1e-13)
    # the high-frequency pairs are exactly i <= 25, the low ones i >= 50 here
    assert np.flatnonzero(hi).max() == 25 and np.flatnonzero(lo).min() == 50


def test_yarn_overextrapolated_dims():
    """"8.3 长上下文技术", section 8.3.2: for D=128, training length 4096 the pairs
    from about d=45 upward never finish one turn (r <= 1), so YaRN with alpha=1
    interpolates them fully (theta/s) while pairs below keep some extrapolation."""
    D, s, Ltr = 128, 40.0, 4096
    plain, _ = oracle.rope_theta_fp64("plain", D)
    yarn, _ = oracle.rope_theta_fp64("yarn", D, scale=s, original_max_pos=Ltr)
    full = np.isclose(yarn, plain / s, rtol=1e-14, atol=0)
    first_full = int(np.flatnonzero(full).min())
    assert full[first_full:].all()
    # the turn count crosses 1 between pair 45 and 46 (45.03 in the page's terms)
    pin("overextrap_d_lo", first_full - 1)


def test_yarn_attention_scale():
    """"Long Context: RoPE / YaRN / NTK / MLA", section 6.3: s=8 gives
    sqrt(1/t) about 1.21 and t about 0.68; mscale is 1 for s <= 1."""
    _, ms = oracle.rope_theta_fp64("yarn", 128, scale=8.0, original_max_pos=8192)
    pin("yarn_mscale_s8", ms)
    pin("yarn_t_s8", 1.0 / ms ** 2)
    _, ms1 = oracle.rope_theta_fp64("yarn", 128, scale=1.0, original_max_pos=8192)
    assert ms1 == 1.0
    _, ms16 = oracle.rope_theta_fp64("yarn", 128, scale=16.0, original_max_pos=8192)
    # ln 16 = 4 ln 2
    assert math.isclose(ms16, 1 + 0.4 * math.log(2), rel_tol=1e-15)


def test_table_is_rounded_fp64():
    """The fp32 table is the fp64 value rounded once to nearest (no midpoint hits
    for the workloads' settings)."""
    for w in workloads.WORKLOADS.values():
        th, ms64 = oracle.rope_theta_fp64(w.mode, w.D, w.base, w.scale, w.original_max_pos,
                                          w.alpha, w.beta)
        t, ms, flags = oracle.rope_table(w.mode, w.D, w.base, w.scale, w.original_max_pos,
                                         w.alpha, w.beta)
        assert flags.sum() == 0, w.name
        for a, b in zip(t, th):
            up, dn = np.nextafter(a, np.float32(np.inf)), np.nextafter(a, np.float32(-np.inf))
            assert abs(float(a) - b) <= min(abs(float(up) - b), abs(float(dn) - b))
        assert abs(float(ms) - ms64) <= 2.0 ** -24 * ms64


def test_midpoint_flag_marks_fp32_midpoints():
    """The flag that exempts a table entry from the bit-exact comparison is set
    exactly where the fp64 value sits on an fp32 rounding midpoint.  With the
    per-pair factor mode theta'_0 = 1 / lambda_0, so lambda_0 = 1 / v puts v
    (to within a few fp64 ulps) into entry 0: a midpoint must flag, and values
    2^-30 (relative) to either side, or an fp32 number itself, must not."""
    D = 64
    for f in (np.float32(1.5), np.float32(0.01), np.float32(3.0517578125e-05)):
        up = np.nextafter(f, np.float32(np.inf))
        mid = 0.5 * (float(f) + float(up))
        cases = [(mid, 1), (mid * (1 + 2.0 ** -30), 0), (mid * (1 - 2.0 ** -30), 0),
                 (float(f), 0), (float(up), 0)]
        for v, expect in cases:
            lam = np.ones(D // 2)
            lam[0] = 1.0 / v
            th, _ = oracle.rope_theta_ext("factors", D, factors=lam)
            assert abs(th[0] - v) <= 4 * np.spacing(v)
            t, ms, flags = oracle.rope_table("factors", D, factors=lam)
            assert flags[0] == expect, (float(f), v)
            assert flags[1:].sum() == 0


# --------------------------------------------------------------------------
# rotation
# --------------------------------------------------------------------------

def test_window_angle_table_d64():
    """"长上下文外推", sections 5.2, 6.1 and 6.2 (d=64, a 4096-position training
    window): each pair's frequency, the angle it covers over the window and the
    turns that makes; the slowest pair's cos / sin at the window's end (taken
    from the oracle's rotation of a unit pair at position 4095); and its angle
    at position 8191, whose sin / cos the page takes at the angle rounded to
    the printed 63 degrees."""
    pins = load_pins()

    def near(name, got):
        val, tol, src = pins[name]
        assert abs(got - val) <= tol, (name, got, val, src)

    table, ms, _ = oracle.rope_table("plain", 64)
    near("d64_i8_freq", float(table[8]))
    near("d64_i24_freq", float(table[24]))
    for i in (0, 8, 16, 24, 31):
        rad = 4096 * float(table[i])
        if "d64_i%d_window_rad" % i in pins:
            near("d64_i%d_window_rad" % i, rad)
        near("d64_i%d_window_turns" % i, rad / (2 * math.pi))
    x = np.zeros((1, 64), dtype=np.float32)
    x[0, 31] = 1.0                                  # unit vector on pair 31's first component
    y = oracle.rotate_rows(x, np.array([4095]), table, ms, "half")
    near("d64_i31_window_cos", y[0, 31])
    near("d64_i31_window_sin", y[0, 63])
    rad = 8191 * float(table[31])
    near("d64_i31_pos8191_rad", rad)
    near("d64_i31_pos8191_deg", math.degrees(rad))
    deg = round(math.degrees(rad))
    near("d64_i31_pos8191_sin", math.sin(math.radians(deg)))
    near("d64_i31_pos8191_cos", math.cos(math.radians(deg)))


@pytest.mark.parametrize("pairing", ["half", "interleaved"])
def test_homework_angles(pairing):
    """"长上下文外推", homework 2: base 1e4, d=4, m=100: pair 0 turns by 100 rad,
    pair 1 by 1 rad.  The rotated unit vector must be (cos a, sin a)."""
    table, ms, _ = oracle.rope_table("plain", 4)
    for i, name in ((0, "angle_m100_i0_d4"), (1, "angle_m100_i1_d4")):
        p, q = (i, i + 2) if pairing == "half" else (2 * i, 2 * i + 1)
        x = np.zeros((1, 4), dtype=np.float32)
        x[0, p] = 1.0
        y = oracle.rotate_rows(x, np.array([100]), table, ms, pairing)[0]
        a = 100 * float(table[i])          # the angle the fp32 table implies
        assert abs(y[p] - math.cos(a)) < 1e-12 and abs(y[q] - math.sin(a)) < 1e-12
        # the other pair is untouched
        others = [d for d in range(4) if d not in (p, q)]
        assert np.all(y[others] == 0.0)
        pin(name, a)


def test_relative_position_demo_15deg():
    """"长上下文外推", section 4.2: q = k = (1, 1), unit angle 15 deg: positions
    (2,5), (10,13), (0,3) give the same dot product 2 cos 45 deg = sqrt 2, and
    (2,6) gives 2 cos 60 deg = 1."""
    table = np.array([math.pi / 12], dtype=np.float32)
    v = np.ones((1, 2), dtype=np.float32)
    t64 = float(table[0])

    def dot(m, n):
        a = oracle.rotate_rows(v, np.array([m]), table, 1.0)[0]
        b = oracle.rotate_rows(v, np.array([n]), table, 1.0)[0]
        return float(a @ b)

    for m, n in ((2, 5), (10, 13), (0, 3)):
        assert abs(dot(m, n) - 2 * math.cos(3 * t64)) < 1e-12
        assert abs(dot(m, n) - math.sqrt(2)) < 1e-6   # table holds 15 deg in fp32
    assert abs(dot(2, 6) - 2 * math.cos(4 * t64)) < 1e-12
    assert abs(dot(2, 6) - 1.0) < 1e-6


@pytest.mark.parametrize("mode", ["plain", "pi", "ntk", "yarn"])
@pytest.mark.parametrize("pairing", ["half", "interleaved"])
def test_rotation_invariants(mode, pairing):
    """"Long Context: RoPE / YaRN / NTK / MLA", section 2.2: <R_m q, R_n k> depends
    on n - m only; rotation keeps norms (times mscale, section 6.4)."""
    D = 128
    table, ms, _ = oracle.rope_table(mode, D, scale=8.0, original_max_pos=8192)
    rng = np.random.default_rng(1)
    q = rng.standard_normal((1, D)).astype(np.float32)
    k = rng.standard_normal((1, D)).astype(np.float32)
    for m, n, t in ((5, 900, 12345), (70000, 3, 40000), (131071, 131000, -131000)):
        a = oracle.rotate_rows(q, np.array([m]), table, ms, pairing)[0]
        b = oracle.rotate_rows(k, np.array([n]), table, ms, pairing)[0]
        a2 = oracle.rotate_rows(q, np.array([m + t]), table, ms, pairing)[0]
        b2 = oracle.rotate_rows(k, np.array([n + t]), table, ms, pairing)[0]
        assert abs(a @ b - a2 @ b2) <= 1e-10 * np.linalg.norm(a) * np.linalg.norm(b)
        assert math.isclose(np.linalg.norm(a), float(ms) * np.linalg.norm(q.astype(np.float64)),
                            rel_tol=1e-13)


def test_pairings_are_a_fixed_permutation():
    """"Long Context: RoPE / YaRN / NTK / MLA", section 2.4: half-split and
    interleaved pairing differ by a fixed permutation of the dimensions."""
    D = 64
    table, ms, _ = oracle.rope_table("yarn", D, scale=4.0, original_max_pos=2048)
    perm = np.empty(D, dtype=np.int64)        # interleaved slot -> half slot
    perm[0::2] = np.arange(D // 2)
    perm[1::2] = np.arange(D // 2) + D // 2
    rng = np.random.default_rng(2)
    x = rng.standard_normal((16, D)).astype(np.float32)
    pos = rng.integers(0, 100000, 16)
    yh = oracle.rotate_rows(x, pos, table, ms, "half")
    yi = oracle.rotate_rows(x[:, perm], pos, table, ms, "interleaved")
    np.testing.assert_array_equal(yi, yh[:, perm])


def test_rotation_plain_reduces_to_complex_multiply():
    """Section 2.1: the rotation is the complex product x * e^{i m theta}
    (checked against numpy's complex exponential on a pair at large m)."""
    D = 128
    table, ms, _ = oracle.rope_table("plain", D)
    rng = np.random.default_rng(3)
    x = rng.standard_normal((4, D)).astype(np.float32)
    pos = np.array([0, 1, 65537, 131071])
    y = oracle.rotate_rows(x, pos, table, ms, "interleaved")
    z = (x[:, 0::2].astype(np.float64) + 1j * x[:, 1::2]) * np.exp(
        1j * pos[:, None] * table.astype(np.float64)[None, :])
    np.testing.assert_allclose(y[:, 0::2], z.real, atol=1e-11)
    np.testing.assert_allclose(y[:, 1::2], z.imag, atol=1e-11)


# --------------------------------------------------------------------------
# masks
# --------------------------------------------------------------------------

def test_sliding_window_mask_worked_example():
    """"Long Context: RoPE / YaRN / NTK / MLA", section 10.1: L=8, W=4 table."""
    golden = np.array(load_mask("swa_mask_L8_W4.txt"))
    np.testing.assert_array_equal(oracle.mask(8, True, 4, 0), golden)


def test_causal_and_degenerate_masks():
    L = 37
    tri = np.tril(np.ones((L, L), dtype=bool))
    np.testing.assert_array_equal(oracle.mask(L, True, 0, 0), tri)
    np.testing.assert_array_equal(oracle.mask(L, True, L, 0), tri)       # W >= L
    np.testing.assert_array_equal(oracle.mask(L, True, 5, L), tri)       # S >= L
    np.testing.assert_array_equal(oracle.mask(L, False, 0, 0), np.ones((L, L), dtype=bool))
    np.testing.assert_array_equal(oracle.mask(L, True, 1, 0), np.eye(L, dtype=bool))


def test_sink_plus_window_cache_size():
    """"Long Context: RoPE / YaRN / NTK / MLA", section 10.2: with S sinks and a
    window W every late query sees exactly S + W keys, always including keys
    0..S-1 and its own W most recent keys."""
    L, W, S = 64, 8, 4
    m = oracle.mask(L, True, W, S)
    for i in range(W + S, L):
        assert m[i].sum() == S + W
        assert m[i, :S].all() and m[i, i - W + 1:i + 1].all()
    # the first rows are causal: nothing is dropped before the cache fills
    for i in range(W):
        assert m[i, :i + 1].all() and m[i].sum() == i + 1


def test_visible_pair_count():
    """The attention work counter: brute-force mask counts, the closed form
    N*W - W(W-1)/2, and "长上下文外推" section 13.1's figure (W=4096 at N=128K:
    about 524M dot products, within the page's approximation)."""
    for L, W, S in ((1, 0, 0), (37, 0, 0), (37, 5, 0), (37, 5, 3), (64, 8, 4), (100, 99, 2),
                    (100, 100, 7), (100, 3, 100)):
        assert workloads.visible_pairs(L, True, W, S) == oracle.mask(L, True, W, S).sum()
    N, W = 128000, 4096
    exact = workloads.visible_pairs(N, True, W, 0)
    assert exact == N * W - W * (W - 1) // 2
    assert abs(exact - 524e6) / 524e6 < 0.02
    assert workloads.visible_pairs(65536, True, 4096, 4) == 260294650


# --------------------------------------------------------------------------
# attention
# --------------------------------------------------------------------------

def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape).astype(np.float32)


def _rotated(x, table, ms, pairing, pos_offset=0):
    B, H, L, D = x.shape
    pos = np.tile(np.arange(L) + pos_offset, B * H)
    return oracle.rotate_rows(x.reshape(-1, D), pos, table, ms, pairing).reshape(B, H, L, D)


@pytest.mark.parametrize("causal,W,S", [(True, 0, 0), (True, 7, 0), (True, 7, 3), (False, 0, 0)])
def test_attention_matches_torch_sdpa_fp64(causal, W, S):
    """Reduction to a library routine: with the oracle's rotated q/k (pinned above),
    the attention output equals torch's fp64 scaled_dot_product_attention with the
    same boolean mask and scale ("Long Context: RoPE / YaRN / NTK / MLA", 2.4)."""
    B, Hq, Hkv, L, D = 2, 4, 2, 45, 64
    table, ms, _ = oracle.rope_table("yarn", D, scale=4.0, original_max_pos=16)
    q, k, v = _rand((B, Hq, L, D), 1), _rand((B, Hkv, L, D), 2), _rand((B, Hkv, L, D), 3)
    o, lse = oracle.attn_full(q, k, v, table, ms, "half", 0, causal, W, S, scale=0.3)
    qr = torch.from_numpy(_rotated(q, table, ms, "half"))
    kr = torch.from_numpy(_rotated(k, table, ms, "half")).repeat_interleave(Hq // Hkv, dim=1)
    vv = torch.from_numpy(v.astype(np.float64)).repeat_interleave(Hq // Hkv, dim=1)
    m = torch.from_numpy(oracle.mask(L, causal, W, S))
    ref = torch.nn.functional.scaled_dot_product_attention(qr, kr, vv, attn_mask=m, scale=0.3)
    np.testing.assert_allclose(o, ref.numpy(), atol=1e-12, rtol=0)
    # lse = max + ln sum exp(s - max) over the visible keys, evaluated in numpy
    # fp64 on numpy's own matmul of the rotated operands
    logits = np.where(m.numpy(), np.matmul(qr.numpy(), np.swapaxes(kr.numpy(), -1, -2)) * 0.3,
                      -np.inf)
    mx = logits.max(axis=-1, keepdims=True)
    ref_lse = mx[..., 0] + np.log(np.exp(logits - mx).sum(axis=-1))
    np.testing.assert_allclose(lse, ref_lse, atol=1e-12, rtol=0)


def test_attention_equals_online_softmax_blocks():
    """"8.3 长上下文技术", section 8.3.4: blockwise online softmax (running max and
    sum with rescaling) gives exactly softmax attention.  An independent blockwise
    loop over 16-key blocks agrees with the oracle to 1e-12."""
    B, H, L, D = 1, 2, 70, 32
    table, ms, _ = oracle.rope_table("ntk", D, scale=2.0)
    q, k, v = _rand((B, H, L, D), 4), _rand((B, H, L, D), 5), _rand((B, H, L, D), 6)
    o, lse = oracle.attn_full(q, k, v, table, ms, "interleaved", 0, True, 20, 2)
    qr, kr = _rotated(q, table, ms, "interleaved"), _rotated(k, table, ms, "interleaved")
    vis = oracle.mask(L, True, 20, 2)
    sc = 1 / math.sqrt(D)
    for h in range(H):
        for i in range(L):
            mrun, lrun, acc = -np.inf, 0.0, np.zeros(D)
            for j0 in range(0, L, 16):
                js = [j for j in range(j0, min(L, j0 + 16)) if vis[i, j]]
                if not js:
                    continue
                s = np.array([sc * qr[0, h, i] @ kr[0, h, j] for j in js])
                mnew = max(mrun, s.max())
                corr = math.exp(mrun - mnew) if mrun > -np.inf else 0.0
                p = np.exp(s - mnew)
                lrun = lrun * corr + p.sum()
                acc = acc * corr + p @ v[0, h, js].astype(np.float64)
                mrun = mnew
            np.testing.assert_allclose(o[0, h, i], acc / lrun, atol=1e-12, rtol=0)
            assert abs(lse[0, h, i] - (mrun + math.log(lrun))) < 1e-12


def test_attention_special_cases():
    """Closed-form special cases of softmax attention."""
    D = 16
    table, ms, _ = oracle.rope_table("plain", D)
    # L = 1: the only key is itself, o = v_0, lse = its logit
    q, k, v = _rand((1, 1, 1, D), 7), _rand((1, 1, 1, D), 8), _rand((1, 1, 1, D), 9)
    o, lse = oracle.attn_full(q, k, v, table, ms)
    np.testing.assert_allclose(o[0, 0, 0], v[0, 0, 0], atol=1e-15)
    qr, kr = _rotated(q, table, ms, "half"), _rotated(k, table, ms, "half")
    assert abs(lse[0, 0, 0] - qr[0, 0, 0] @ kr[0, 0, 0] / 4.0) < 1e-12
    # W = 1 (no sinks): each query sees only itself
    L = 33
    q, k, v = _rand((1, 2, L, D), 10), _rand((1, 2, L, D), 11), _rand((1, 2, L, D), 12)
    o, _ = oracle.attn_full(q, k, v, table, ms, window=1)
    np.testing.assert_allclose(o, v.astype(np.float64), atol=1e-14)
    # q = 0: uniform weights over the visible keys, lse = ln(count)
    q0 = np.zeros((1, 2, L, D), dtype=np.float32)
    o, lse = oracle.attn_full(q0, k, v, table, ms, window=5, sinks=2)
    vis = oracle.mask(L, True, 5, 2)
    for i in range(L):
        np.testing.assert_allclose(o[0, :, i], v[0].astype(np.float64)[:, vis[i]].mean(axis=1), atol=1e-14)
        assert abs(lse[0, 0, i] - math.log(vis[i].sum())) < 1e-14
    # identical keys at every position under mode NONE: uniform weights again
    tab0, ms0, _ = oracle.rope_table("none", D)
    kc = np.repeat(_rand((1, 1, 1, D), 13), L, axis=2)
    o, _ = oracle.attn_full(_rand((1, 1, L, D), 14), kc, v[:, :1], tab0, ms0)
    for i in range(L):
        np.testing.assert_allclose(o[0, 0, i], v[0, 0, :i + 1].astype(np.float64).mean(axis=0), atol=1e-13)


def test_gqa_equals_replicated_heads_and_degenerate_windows():
    """GQA (query head h reads kv head h // G) equals MHA on replicated K/V; a
    window or sink count of at least L is plain causal attention."""
    B, Hq, Hkv, L, D = 1, 6, 2, 40, 32
    table, ms, _ = oracle.rope_table("pi", D, scale=2.0)
    q, k, v = _rand((B, Hq, L, D), 15), _rand((B, Hkv, L, D), 16), _rand((B, Hkv, L, D), 17)
    o_gqa, l_gqa = oracle.attn_full(q, k, v, table, ms)
    o_mha, l_mha = oracle.attn_full(q, np.repeat(k, 3, axis=1), np.repeat(v, 3, axis=1), table, ms)
    np.testing.assert_array_equal(o_gqa, o_mha)
    np.testing.assert_array_equal(l_gqa, l_mha)
    o_w, _ = oracle.attn_full(q, k, v, table, ms, window=L)
    o_s, _ = oracle.attn_full(q, k, v, table, ms, window=3, sinks=L)
    np.testing.assert_array_equal(o_w, o_gqa)
    np.testing.assert_array_equal(o_s, o_gqa)


def test_attention_depends_on_relative_positions_only():
    """Section 2.2 carried through softmax: shifting every position by t leaves the
    attention output unchanged (up to rounding)."""
    B, H, L, D = 1, 2, 30, 64
    table, ms, _ = oracle.rope_table("yarn", D, scale=8.0, original_max_pos=64)
    q, k, v = _rand((B, H, L, D), 18), _rand((B, H, L, D), 19), _rand((B, H, L, D), 20)
    o0, l0 = oracle.attn_full(q, k, v, table, ms, pos_offset=0, window=9, sinks=1)
    o1, l1 = oracle.attn_full(q, k, v, table, ms, pos_offset=100000, window=9, sinks=1)
    np.testing.assert_allclose(o0, o1, atol=1e-9)
    np.testing.assert_allclose(l0, l1, atol=1e-9)


def test_invalid_arguments_rejected():
    with pytest.raises(ValueError):
        oracle.rope_table("plain", 63)
    with pytest.raises(ValueError):
        oracle.rope_table("yarn", 64, scale=4.0, alpha=32.0, beta=1.0)
    k = np.zeros((1, 2, 4, 8), dtype=np.float32)
    table, ms, _ = oracle.rope_table("plain", 8)
    with pytest.raises(ValueError):   # Hq not a multiple of Hkv
        oracle.attn_rows(np.zeros((1, 8), np.float32), [0], [0], [0], k, k, 3, table, ms)
    with pytest.raises(ValueError):   # window without causal
        oracle.attn_rows(np.zeros((1, 8), np.float32), [0], [0], [0], k, k, 2, table, ms,
                         causal=False, window=2)


# --------------------------------------------------------------------------
# length-dependent table variants
# --------------------------------------------------------------------------

def test_dynamic_ntk_keeps_short_sequences_plain():
    """"AI Day 9: 长上下文技术", RoPE extension list item 4 (Dynamic NTK): the base
    follows the actual sequence length and short sequences are unchanged."""
    for seq in (1, 4096, 8192):
        t, ms, _ = oracle.rope_table("dynamic_ntk", 128, original_max_pos=8192, seq_len=seq)
        plain, _, _ = oracle.rope_table("plain", 128)
        np.testing.assert_array_equal(t, plain)
        assert ms == 1.0


def test_dynamic_ntk_base_for_8k_to_128k():
    """With the actual length 131072 over a training length of 8192 the dynamic
    base is the NTK-aware base for s = 16: about 1.7e5 ("长上下文推理" plumephp NTK
    comment); longer sequences get lower low frequencies."""
    th, _ = oracle.rope_theta_ext("dynamic_ntk", 128, original_max_pos=8192, seq_len=131072)
    pin("ntk_b1e4_d128_s16", ntk_base_from_table(th, 128))
    prev = None
    for seq in (16384, 32768, 65536, 131072):
        th, _ = oracle.rope_theta_ext("dynamic_ntk", 128, original_max_pos=8192, seq_len=seq)
        assert th[0] == 1.0
        if prev is not None:
            assert (th[1:] < prev[1:]).all()
        prev = th


def test_factor_tables():
    """"Long Context: RoPE / YaRN / NTK / MLA", 7.3: theta'_i = theta_i / lambda_i.
    lambda = s everywhere is PI (7.4's uniform row), lambda = 1 is plain, the
    inverse YaRN multipliers reproduce YaRN (7.4: a three-segment ramp is one
    choice of lambda), and 7.4's short-context rescue switches to the short table
    while the actual length is within the training length."""
    D, s = 128, 8.0
    plain, _, _ = oracle.rope_table("plain", D)
    pi, _, _ = oracle.rope_table("pi", D, scale=s)
    t, ms, _ = oracle.rope_table("factors", D, factors=np.full(D // 2, s), seq_len=10 ** 6)
    np.testing.assert_array_equal(t, pi)
    assert ms == 1.0
    t, _, _ = oracle.rope_table("factors", D, factors=np.ones(D // 2), seq_len=10 ** 6)
    np.testing.assert_array_equal(t, plain)
    th, _ = oracle.rope_theta_fp64("plain", D)
    yarn, _ = oracle.rope_theta_fp64("yarn", D, scale=s, original_max_pos=8192)
    lam = th / yarn
    tf, _ = oracle.rope_theta_ext("factors", D, factors=lam, seq_len=10 ** 6)
    np.testing.assert_allclose(tf, yarn, rtol=1e-15)
    short = np.ones(D // 2)
    long_ = np.full(D // 2, 4.0)
    ts, _, _ = oracle.rope_table("factors", D, original_max_pos=4096, seq_len=4096,
                                 factors=long_, factors_short=short)
    tl, _, _ = oracle.rope_table("factors", D, original_max_pos=4096, seq_len=4097,
                                 factors=long_, factors_short=short)
    np.testing.assert_array_equal(ts, plain)
    np.testing.assert_array_equal(tl, oracle.rope_table("pi", D, scale=4.0)[0])
    with pytest.raises(ValueError):
        oracle.rope_table("factors", D, factors=np.zeros(D // 2), seq_len=1)
    with pytest.raises(ValueError):
        oracle.rope_table("dynamic_ntk", D, seq_len=0)


# --------------------------------------------------------------------------
# Chunked prefill, decode and the StreamingLLM cache ("Long Context: RoPE /
# YaRN / NTK / MLA", section 10.3): the oracle evaluates query rows at any index
# into the key arrays; these pin what the decode-time readings compute.

def test_chunked_rows_equal_prefill_rows():
    """A query chunk evaluated against only the keys up to its end equals the
    same rows of the full causal prefill (keys beyond a causal row are masked)."""
    B, Hq, Hkv, L, D = 1, 4, 2, 50, 32
    table, ms, _ = oracle.rope_table("yarn", D, scale=4.0, original_max_pos=16)
    q, k, v = _rand((B, Hq, L, D), 40), _rand((B, Hkv, L, D), 41), _rand((B, Hkv, L, D), 42)
    o_full, l_full = oracle.attn_full(q, k, v, table, ms, window=11, sinks=2)
    a, b = 17, 33
    hh, ii = np.meshgrid(np.arange(Hq), np.arange(a, b), indexing="ij")
    o, lse = oracle.attn_rows(q[0][hh.ravel(), ii.ravel()], np.zeros(hh.size, np.int64),
                              hh.ravel(), ii.ravel(), k[:, :, :b], v[:, :, :b], Hq, table, ms,
                              window=11, sinks=2)
    np.testing.assert_array_equal(o.reshape(Hq, b - a, D), o_full[0, :, a:b])
    np.testing.assert_array_equal(lse.reshape(Hq, b - a), l_full[0, :, a:b])


def test_streaming_cache_without_sinks_is_a_sliding_window():
    """With no sink tokens, a StreamingLLM step (the W most recent un-rotated keys
    re-indexed to positions 0..W-1, the new token at position W) sees the same
    keys at the same relative distances as sliding-window attention over the
    absolute sequence with a window of W + 1 (the query included), so by the
    relative-position property of RoPE (section 2.2) the outputs agree."""
    H, N, D, W = 2, 64, 32, 12
    table, ms, _ = oracle.rope_table("yarn", D, scale=8.0, original_max_pos=16)
    q, k, v = _rand((1, H, N, D), 43), _rand((1, H, N, D), 44), _rand((1, H, N, D), 45)
    o_abs, l_abs = oracle.attn_full(q, k, v, table, ms, window=W + 1)
    for t in (W, W + 5, N - 1):
        kc, vc = k[:, :, t - W:t + 1], v[:, :, t - W:t + 1]
        o, lse = oracle.attn_rows(q[0, :, t], np.zeros(H, np.int64), np.arange(H),
                                  np.full(H, W), kc, vc, H, table, ms)
        np.testing.assert_allclose(o, o_abs[0, :, t], atol=1e-10, rtol=0)
        np.testing.assert_allclose(lse, l_abs[0, :, t], atol=1e-10, rtol=0)


def test_streaming_cache_before_eviction_is_plain_causal():
    """While the sequence fits in S + W entries nothing is evicted, every key keeps
    its index as position, and a decode step equals the last causal row."""
    H, N, D = 1, 20, 16
    table, ms, _ = oracle.rope_table("plain", D)
    q, k, v = _rand((1, H, N, D), 46), _rand((1, H, N, D), 47), _rand((1, H, N, D), 48)
    o_full, _ = oracle.attn_full(q, k, v, table, ms)
    o, _ = oracle.attn_rows(q[0, :, N - 1], [0], [0], [N - 1], k, v, H, table, ms)
    np.testing.assert_array_equal(o[0], o_full[0, 0, N - 1])


# --------------------------------------------------------------------------
# Split-KV partial attention and the (O, LSE) merge ("8.3 长上下文技术", 8.3.4
# online softmax, 8.3.5 Ring Attention step 3).

@pytest.mark.parametrize("causal,W,S", [(True, 0, 0), (True, 9, 3), (False, 0, 0)])
def test_merge_of_key_partitions_is_full_attention(causal, W, S):
    """Partial results over a partition of the keys (some parts empty for some
    rows) merge to the full attention result: the softmax identity behind
    split-KV and ring attention."""
    B, Hq, Hkv, L, D = 1, 4, 2, 41, 32
    table, ms, _ = oracle.rope_table("yarn", D, scale=4.0, original_max_pos=16)
    q, k, v = _rand((B, Hq, L, D), 50), _rand((B, Hkv, L, D), 51), _rand((B, Hkv, L, D), 52)
    o_full, l_full = oracle.attn_full(q, k, v, table, ms, "half", 0, causal, W, S)
    hh, ii = np.meshgrid(np.arange(Hq), np.arange(L), indexing="ij")
    rows = dict(q_rows=q[0][hh.ravel(), ii.ravel()], row_b=np.zeros(hh.size, np.int64),
                row_h=hh.ravel(), row_i=ii.ravel(), k=k, v=v, Hq=Hq, table=table, mscale=ms,
                causal=causal, window=W, sinks=S)
    cuts = [0, 5, 6, 20, 33, 41]
    parts = [oracle.attn_rows(**rows, k_begin=a, k_end=b) for a, b in zip(cuts, cuts[1:])]
    o, lse = oracle.merge(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
    np.testing.assert_allclose(o.reshape(Hq, L, D), o_full[0], atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse.reshape(Hq, L), l_full[0], atol=1e-12, rtol=0)
    # a part with no visible key is the empty sum
    assert np.isneginf(parts[-1][1][:5]).all() or not causal


def test_merge_closed_forms():
    rng = np.random.default_rng(53)
    o1, o2 = rng.standard_normal((2, 3, 8))
    l1 = rng.standard_normal(3)
    # one part: identity
    o, lse = oracle.merge(o1[None], l1[None])
    np.testing.assert_array_equal(o, o1)
    np.testing.assert_array_equal(lse, l1)
    # equal weights: the mean, lse + ln 2
    o, lse = oracle.merge(np.stack([o1, o2]), np.stack([l1, l1]))
    np.testing.assert_allclose(o, (o1 + o2) / 2, atol=1e-15)
    np.testing.assert_allclose(lse, l1 + math.log(2), atol=1e-15)
    # an empty part changes nothing; all parts empty -> o = 0, lse = -inf
    o, lse = oracle.merge(np.stack([o1, o2]), np.stack([l1, np.full(3, -np.inf)]))
    np.testing.assert_array_equal(o, o1)
    np.testing.assert_array_equal(lse, l1)
    o, lse = oracle.merge(np.stack([o1, o2]), np.full((2, 3), -np.inf))
    assert (o == 0).all() and np.isneginf(lse).all()
    # weights e^{lse_s}: a part 10 nats heavier dominates with weight 1/(1+e^-10)
    o, _ = oracle.merge(np.stack([o1, o2]), np.stack([l1 + 10.0, l1]))
    w = 1.0 / (1.0 + math.exp(-10.0))
    np.testing.assert_allclose(o, w * o1 + (1 - w) * o2, atol=1e-14)
    # order of the parts does not matter
    oa, la = oracle.merge(np.stack([o1, o2]), np.stack([l1, l1 - 1]))
    ob, lb = oracle.merge(np.stack([o2, o1]), np.stack([l1 - 1, l1]))
    np.testing.assert_allclose(oa, ob, atol=1e-15)
    np.testing.assert_allclose(la, lb, atol=1e-15)


# --------------------------------------------------------------------------
# Decoupled RoPE ("Long Context: RoPE / YaRN / NTK / MLA", 9.5 and 9.7; A.1):
# q = [q_C ; RoPE(q_R)], k^(h) = [k_C^(h) ; RoPE(k_R)] with k_R shared by all
# heads, scores scaled by 1/sqrt(d_C + d_R).

def _mla_inputs(B, Hq, Hkv, L, Dc, Dr, Dv, seed):
    return (_rand((B, Hq, L, Dc + Dr), seed), _rand((B, Hkv, L, Dc), seed + 1),
            _rand((B, L, Dr), seed + 2), _rand((B, Hkv, L, Dv), seed + 3))


def _all_rows(B, Hq, L):
    bb, hh, ii = np.meshgrid(np.arange(B), np.arange(Hq), np.arange(L), indexing="ij")
    return bb.ravel(), hh.ravel(), ii.ravel()


def test_mla_without_nope_part_is_shared_key_attention():
    """With d_C = 0 every head attends with the one shared rotary key: the
    standard oracle with a single kv head (GQA over all heads)."""
    B, Hq, L, Dr = 1, 4, 33, 32
    table, ms, _ = oracle.rope_table("yarn", Dr, scale=4.0, original_max_pos=8)
    q, kc, kr, v = _mla_inputs(B, Hq, 1, L, 0, Dr, Dr, 60)
    bb, hh, ii = _all_rows(B, Hq, L)
    o, lse = oracle.attn_rows_mla(q.reshape(-1, Dr), bb, hh, ii, kc, kr, v, Hq, table, ms,
                                  window=9, sinks=2)
    ref_o, ref_l = oracle.attn_full(q, kr[:, None], v, table, ms, window=9, sinks=2)
    np.testing.assert_allclose(o.reshape(B, Hq, L, Dr), ref_o, atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse.reshape(B, Hq, L), ref_l, atol=1e-12, rtol=0)


@pytest.mark.parametrize("pairing,Hkv", [("half", 4), ("interleaved", 4), ("half", 2)])
def test_mla_matches_torch_sdpa_on_concatenated_vectors(pairing, Hkv):
    """Reduction to a library routine: torch's fp64 scaled_dot_product_attention
    on explicitly concatenated [q_C ; rotated q_R] and [k_C ; rotated k_R] (the
    rotation pinned above, mscale on the rotated parts), value dim d_v != d_qk;
    with Hkv < Hq, query head h takes the k_C and v of head h // G (K/V
    replicated G times before the library call)."""
    B, Hq, L, Dc, Dr, Dv = 2, 4, 29, 48, 16, 24
    G = Hq // Hkv
    table, ms, _ = oracle.rope_table("yarn", Dr, scale=8.0, original_max_pos=4)
    assert ms > 1.0
    q, kc, kr, v = _mla_inputs(B, Hq, Hkv, L, Dc, Dr, Dv, 61)
    bb, hh, ii = _all_rows(B, Hq, L)
    o, lse = oracle.attn_rows_mla(q.reshape(-1, Dc + Dr), bb, hh, ii, kc, kr, v, Hq, table, ms,
                                  pairing, causal=True, window=11, sinks=3)
    qr = oracle.rotate_rows(q[..., Dc:].reshape(-1, Dr), np.tile(np.arange(L), B * Hq), table,
                            ms, pairing).reshape(B, Hq, L, Dr)
    krr = oracle.rotate_rows(kr.reshape(-1, Dr), np.tile(np.arange(L), B), table, ms,
                             pairing).reshape(B, 1, L, Dr)
    qcat = torch.from_numpy(np.concatenate([q[..., :Dc].astype(np.float64), qr], axis=-1))
    kcat = torch.from_numpy(np.concatenate([np.repeat(kc, G, axis=1).astype(np.float64),
                                            np.repeat(krr, Hq, axis=1)], axis=-1))
    m = torch.from_numpy(oracle.mask(L, True, 11, 3))
    ref = torch.nn.functional.scaled_dot_product_attention(
        qcat, kcat, torch.from_numpy(np.repeat(v, G, axis=1).astype(np.float64)), attn_mask=m,
        scale=1.0 / math.sqrt(Dc + Dr))
    np.testing.assert_allclose(o.reshape(B, Hq, L, Dv), ref.numpy(), atol=1e-12, rtol=0)
    logits = (qcat @ kcat.transpose(-1, -2)) / math.sqrt(Dc + Dr)
    ref_l = torch.logsumexp(logits.masked_fill(~m, float("-inf")), dim=-1)
    np.testing.assert_allclose(lse.reshape(B, Hq, L), ref_l.numpy(), atol=1e-12, rtol=0)


def test_mla_relative_positions_only():
    B, Hq, L, Dc, Dr = 1, 2, 20, 32, 32
    table, ms, _ = oracle.rope_table("ntk", Dr, scale=4.0)
    q, kc, kr, v = _mla_inputs(B, Hq, Hq, L, Dc, Dr, 32, 62)
    bb, hh, ii = _all_rows(B, Hq, L)
    a = oracle.attn_rows_mla(q.reshape(-1, Dc + Dr), bb, hh, ii, kc, kr, v, Hq, table, ms)
    b = oracle.attn_rows_mla(q.reshape(-1, Dc + Dr), bb, hh, ii, kc, kr, v, Hq, table, ms,
                             pos_offset=77777)
    np.testing.assert_allclose(a[0], b[0], atol=1e-9)
    np.testing.assert_allclose(a[1], b[1], atol=1e-9)
