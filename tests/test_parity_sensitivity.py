"""The GPU parity comparison is sharp enough to see a kernel that gets its own
arithmetic wrong.

A kernel can make the same mistakes as the oracle's mutants: a mask
off-by-one, a wrong pairing or rotation sign, mscale on one component only,
the wrong kv head, a missing score scale, bad softmax statistics, a key split
that reads outside its stretch, or a merge that weights its parts wrongly.  For each
such mistake, a copy of the oracle with it planted stands in for the kernel.
It is compared with the unchanged oracle by the GPU tests' own comparison
(test_gpu_attn.compare: max-abs 2e-2 beyond the output's rounding, mean-abs
2e-3, LSE 2e-2), on inputs drawn like the GPU tests' small cases.  At least one
of those cases must fail the comparison.  Everything runs on the CPU.  The
RoPE table is the unchanged oracle's on both sides, because the kernel takes
its table from the host.
"""
import importlib.util
import os
import sys

import numpy as np
import pytest
import torch

import oracle
from test_gpu_attn import BASE, SMALL, compare, table_of
from test_gpu_decode import W0, oracle_rows, rope_of
from test_gpu_rope import CASES as ROPE_CASES, check_rotation
from test_oracle_mutants import MUTANTS, _copy_oracle
from workloads import make_inputs

# mistakes a kernel could make in its own arithmetic (the table comes from the host)
PREFILL_MUTANTS = [
    "causal_sees_next_key", "causal_hides_diagonal", "window_one_too_wide",
    "sinks_one_too_many", "sinks_seen_by_earlier_queries", "noncausal_hides_future",
    "rotation_first_sign", "rotation_second_sign", "rotation_mscale_one_component",
    "half_pairing_mirrored", "interleaved_pair_reversed", "gqa_heads_interleaved",
    "lse_without_max", "output_not_normalised", "default_scale_one_over_d",
]
# mistakes of the rotate pass (lcx_apply_rope): rotation signs, mscale on one
# component, pairings, and the angle of position m + 1
ROPE_MUTANTS = [
    "rotation_first_sign", "rotation_second_sign", "rotation_mscale_one_component",
    "half_pairing_mirrored", "interleaved_pair_reversed", "position_plus_one",
]
# mistakes of a split-KV launch: a split that reads outside its stretch of keys,
# or a merge that combines the partial results wrongly
SPLIT_MUTANTS = [
    "key_range_start_ignored", "key_range_end_ignored", "merge_equal_weights",
    "merge_lse_without_max", "merge_not_normalised",
]
MLA_MUTANTS = [
    "mla_rope_slice_first", "mla_key_without_mscale", "mla_key_positions_across_batch",
    "mla_heads_interleaved", "mla_lse_without_max", "mla_default_scale_rope_dims",
]

# decoupled-RoPE shapes of the GPU tests (test_gpu_mla.py and the random
# decoupled-RoPE draws, which include batch 2): (B, Dc, Hq, Hkv, L, pairing, W, S)
MLA_CASES = [
    (1, 128, 4, 4, 700, "half", 0, 0),
    (1, 128, 8, 2, 333, "half", 150, 4),
    (1, 128, 2, 2, 257, "interleaved", 0, 0),
    (2, 64, 3, 1, 200, "half", 0, 0),
]


@pytest.fixture(scope="module")
def copies(tmp_path_factory):
    """name -> the oracle package copy with that mistake planted, imported
    under its own module name (its library built in its own folder); the
    "unchanged" copy has none."""
    mods = {}
    names = PREFILL_MUTANTS + SPLIT_MUTANTS + MLA_MUTANTS
    for name in ["unchanged"] + names + [m for m in ROPE_MUTANTS if m not in names]:
        _, file, edits = MUTANTS[name] if name in MUTANTS else ("", "lcx_oracle.c", [])
        dst = str(tmp_path_factory.mktemp("sens_" + name))
        err = _copy_oracle(dst, edits, file)
        assert err is None, err
        pkg = os.path.join(dst, "oracle")
        modname = "oracle_mutant_" + name
        spec = importlib.util.spec_from_file_location(
            modname, os.path.join(pkg, "__init__.py"), submodule_search_locations=[pkg])
        mod = importlib.util.module_from_spec(spec)
        sys.modules[modname] = mod
        spec.loader.exec_module(mod)
        assert os.path.dirname(mod.__file__) == pkg
        mods[name] = mod
    yield mods
    for name in mods:
        sys.modules.pop("oracle_mutant_" + name, None)


def _cases():
    ws = [BASE.with_(**kw) for kw in SMALL.values()]
    return sorted(ws, key=lambda w: w.B * w.Hq * w.L * w.L * w.D)   # cheapest first


_ref_cache = {}


def _prefill(lib, w):
    q, k, v = (t.float().numpy() for t in make_inputs(w, device="cpu"))
    table, ms = table_of(w)
    scale = w.softmax_scale if w.softmax_scale > 0 else None
    return lib.attn_full(q, k, v, table, ms, w.pairing, 0, w.causal, w.window, w.sinks, scale)


def _caught(got, ref, out_bits):
    try:
        compare(got[0], got[1], ref[0], ref[1], out_bits)
    except AssertionError:
        return True
    return False


def test_unchanged_copy_passes_the_comparison(copies):
    """The harness itself: a copy without a planted mistake passes (on the
    cheapest cases), so a failure below comes from the mistake."""
    for w in _cases()[:6]:
        ref = _ref_cache.setdefault(repr(w), _prefill(oracle, w))
        assert not _caught(_prefill(copies["unchanged"], w), ref, 24 if w.dtype == "f32" else 8)
    for case in MLA_CASES[:2]:
        ref = _ref_cache.setdefault(("mla",) + case, _mla(oracle, case))
        assert not _caught(_mla(copies["unchanged"], case), ref, 8)


@pytest.mark.parametrize("name", PREFILL_MUTANTS)
def test_prefill_comparison_sees_kernel_mistake(copies, name):
    for w in _cases():
        key = repr(w)
        if key not in _ref_cache:
            _ref_cache[key] = _prefill(oracle, w)
        got = _prefill(copies[name], w)
        if _caught(got, _ref_cache[key], 24 if w.dtype == "f32" else 8):
            return
    pytest.fail("no GPU small case's comparison sees %r (%s)" % (name, MUTANTS[name][0]))


def _mla(lib, case, seed=11):
    B, Dc, Hq, Hkv, L, pairing, W, S = case
    Dr, Dv = 64, 128
    g = torch.Generator().manual_seed(seed)
    q = torch.randn((B, Hq, L, Dc + Dr), generator=g).bfloat16().float().numpy()
    kc = torch.randn((B, Hkv, L, Dc), generator=g).bfloat16().float().numpy()
    kr = torch.randn((B, L, Dr), generator=g).bfloat16().float().numpy()
    v = torch.randn((B, Hkv, L, Dv), generator=g).bfloat16().float().numpy()
    table, ms, _ = oracle.rope_table("yarn", Dr, scale=8.0, original_max_pos=128)
    bb, hh, ii = np.meshgrid(np.arange(B), np.arange(Hq), np.arange(L), indexing="ij")
    o, lse = lib.attn_rows_mla(q.reshape(-1, Dc + Dr), bb.ravel(), hh.ravel(), ii.ravel(), kc,
                               kr, v, Hq, table, ms, pairing, 0, True, W, S)
    return o, lse


@pytest.mark.parametrize("name", MLA_MUTANTS)
def test_decoupled_rope_comparison_sees_kernel_mistake(copies, name):
    for case in MLA_CASES:
        key = ("mla",) + case
        if key not in _ref_cache:
            _ref_cache[key] = _mla(oracle, case)
        if _caught(_mla(copies[name], case), _ref_cache[key], 8):
            return
    pytest.fail("no decoupled-RoPE case's comparison sees %r (%s)" % (name, MUTANTS[name][0]))


# split-KV shapes of the GPU tests (test_gpu_splitkv.py): (L, Lk, splits, extra)
SPLIT_CASES = [
    (1, 777, 3, {}),
    (4, 5000, 8, dict(window=1000, sinks=4)),
    (2, 900, 5, dict(window=300, sinks=2)),
    (1, 4096, 32, dict(Hq=8, Hkv=2)),
]


def _split(rows_lib, merge_lib, case):
    """Split-KV the way the kernel partitions it (reading 27: split s takes the
    s-th stretch of ceil(n / splits) key tiles of 128, later ones may be empty),
    each split by rows_lib over its key range, combined by merge_lib."""
    L, Lk, splits, extra = case
    w = W0.with_(**extra, L=Lk)
    q_all, k, v = make_inputs(w, device="cpu")
    q = q_all[:, :, Lk - L:]
    rope = rope_of(w)
    B, Hq, _, D = q.shape
    table, ms, _ = oracle.rope_table(rope.mode, D, rope.base, rope.scale, rope.original_max_pos,
                                     rope.alpha, rope.beta, seq_len=Lk)
    bb, hh, ii = (x.ravel() for x in np.meshgrid(np.arange(B), np.arange(Hq), np.arange(L),
                                                 indexing="ij"))
    qr, kk, vv = (t.float().numpy() for t in (q, k, v))
    n_tiles = -(-Lk // 128)
    c = -(-n_tiles // splits) * 128          # keys per split
    parts = [rows_lib.attn_rows(qr.reshape(-1, D), bb, hh, ii + Lk - L, kk, vv, Hq, table, ms,
                                rope.pairing, 0, True, w.window, w.sinks,
                                k_begin=min(Lk, s * c), k_end=min(Lk, (s + 1) * c))
             for s in range(splits)]
    o, lse = merge_lib.merge(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
    ref = oracle_rows(q, k, v, rope, Lk - L, True, w.window, w.sinks)
    return (o.reshape(B, Hq, L, D), lse.reshape(B, Hq, L)), ref


def test_unchanged_split_passes_the_comparison(copies):
    for case in SPLIT_CASES[:2]:
        got, ref = _split(copies["unchanged"], copies["unchanged"], case)
        assert not _caught(got, ref, 8)


@pytest.mark.parametrize("name", SPLIT_MUTANTS)
def test_splitkv_comparison_sees_kernel_mistake(copies, name):
    mod = copies[name]
    for case in SPLIT_CASES:
        rows_lib, merge_lib = (oracle, mod) if name.startswith("merge") else (mod, oracle)
        got, ref = _split(rows_lib, merge_lib, case)
        if _caught(got, ref, 8):
            return
    pytest.fail("no split-KV case's comparison sees %r (%s)" % (name, MUTANTS[name][0]))


def _rotate(lib, case):
    """The rotate pass's output as a kernel would store it (the copy's fp64
    rotation rounded once to the tensor's type), with the unchanged table."""
    B, H, L, D, dt, mode, s, pairing, off = case
    g = torch.Generator().manual_seed(0)
    x = torch.randn((B, H, L, D), generator=g).to(dt)
    rope = rope_of(W0.with_(D=D, mode=mode, scale=s, original_max_pos=2048, pairing=pairing))
    table, ms, _ = oracle.rope_table(mode, D, rope.base, s, 2048, rope.alpha, rope.beta)
    pos = np.tile(np.arange(L) + off, B * H)
    y = lib.rotate_rows(x.float().numpy().reshape(-1, D), pos, table, ms, pairing)
    return x, torch.from_numpy(y.reshape(B, H, L, D)).to(dt), rope, off


def test_unchanged_rotation_passes_the_check(copies):
    for case in ROPE_CASES:
        check_rotation(*_rotate(copies["unchanged"], case))


@pytest.mark.parametrize("name", ROPE_MUTANTS)
def test_rotation_check_sees_kernel_mistake(copies, name):
    for case in ROPE_CASES:
        try:
            check_rotation(*_rotate(copies[name], case))
        except AssertionError:
            return
    pytest.fail("no apply_rope case's check sees %r (%s)" % (name, MUTANTS[name][0]))
