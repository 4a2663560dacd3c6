"""CPU checks of the C-ABI library: it loads, exports what include/lcx.h declares,
its structs match the binding, its host-side table is bit-exact with the oracle,
and malformed arguments are rejected before any device work."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

import ntk_rope_flashattn_b200 as lcx
from ntk_rope_flashattn_b200 import build as lcx_build
import oracle
import workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lcx.h")


@pytest.fixture(scope="module")
def lib():
    lcx_build.build()
    return lcx.load()


def declared_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"LCX_API\s+[\w\s\*]+?\b(lcx_\w+)\s*\(", src)))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert set(names) == set(lcx.EXPORTED)
    out = subprocess.run(["nm", "-D", "--defined-only", lcx.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    for n in names:
        assert n in exported, n
        assert getattr(lib, n) is not None
    # nothing else leaks out of the library
    assert {e for e in exported if e.startswith("lcx")} == set(names)


def test_version_and_status_strings(lib):
    assert lcx.version() == 102
    for st in range(5):
        assert lib.lcx_status_string(st).decode()
    assert lib.lcx_status_string(99).decode() == "unknown status"


def test_struct_layout_matches_header(tmp_path):
    """Offsets and sizes of the C structs, compiled by gcc from include/lcx.h, equal
    the ctypes mirrors the binding uses."""
    src = tmp_path / "layout.c"
    src.write_text(r'''
#include <stdio.h>
#include <stddef.h>
#include "lcx.h"
#define P(T, f) printf(#T "." #f " %zu\n", offsetof(T, f));
int main(void) {
  printf("lcx_rope_params %zu\n", sizeof(lcx_rope_params));
  printf("lcx_attn_args %zu\n", sizeof(lcx_attn_args));
  P(lcx_rope_params, base) P(lcx_rope_params, original_max_pos) P(lcx_rope_params, beta)
  P(lcx_rope_params, seq_len) P(lcx_rope_params, factors) P(lcx_rope_params, factors_short)
  P(lcx_attn_args, dev_status) P(lcx_attn_args, dtype) P(lcx_attn_args, B) P(lcx_attn_args, D)
  P(lcx_attn_args, q_strides) P(lcx_attn_args, o_strides) P(lcx_attn_args, rope)
  P(lcx_attn_args, window) P(lcx_attn_args, sinks) P(lcx_attn_args, softmax_scale)
  P(lcx_attn_args, flags) P(lcx_attn_args, watchdog_ms) P(lcx_attn_args, reserved0)
  P(lcx_attn_args, Lk) P(lcx_attn_args, q_offset) P(lcx_attn_args, Dv)
  P(lcx_attn_args, k_rope) P(lcx_attn_args, k_rope_strides) P(lcx_attn_args, k_rot)
  P(lcx_attn_args, k_rot_bytes)
  return 0;
}
''')
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), str(src), "-o",
                    str(exe)], check=True)
    got = dict(line.rsplit(" ", 1) for line in subprocess.run(
        [str(exe)], capture_output=True, text=True, check=True).stdout.splitlines())
    R, A = lcx._RopeParams, lcx._AttnArgs
    assert int(got["lcx_rope_params"]) == ctypes.sizeof(R)
    assert int(got["lcx_attn_args"]) == ctypes.sizeof(A)
    for key, val in got.items():
        if "." in key:
            T, f = key.split(".")
            assert getattr(R if T == "lcx_rope_params" else A, f).offset == int(val), key


def _params(mode, D, **kw):
    return lcx.RopeParams(mode=mode, head_dim=D, **kw)


TABLE_CASES = [(w.mode, w.D, w.base, w.scale, w.original_max_pos, w.alpha, w.beta)
               for w in workloads.WORKLOADS.values()]
TABLE_CASES += [(m, D, b, s, L, 1.0, 32.0) for m in ("plain", "pi", "ntk", "yarn", "none")
                for D in (2, 4, 64, 80, 96, 128, 256, 512) for b in (1e4, 5e5, 1e6)
                for s in (1.0, 2.0, 4.0, 8.0, 16.0, 40.0) for L in (2048, 8192)
                if not (m == "ntk" and D < 4)]


def test_rope_table_bit_exact_with_oracle(lib):
    """lcx_rope_table (host) equals the oracle's fp32 table bit for bit, for the
    workloads' settings and a sweep of head dims, bases and scales."""
    checked = 0
    for mode, D, base, s, Ltr, a, b in TABLE_CASES:
        ref, ref_ms, flags = oracle.rope_table(mode, D, base, s, Ltr, a, b)
        got, ms = lcx.rope_table(_params(mode, D, base=base, scale=s, original_max_pos=Ltr,
                                         alpha=a, beta=b))
        ok = flags[:-1] == 0
        np.testing.assert_array_equal(got.view(np.uint32)[ok], ref.view(np.uint32)[ok])
        if flags[-1] == 0:
            assert np.float32(ms).view(np.uint32) == np.float32(ref_ms).view(np.uint32)
        checked += int(ok.sum())
    assert checked > 10000


def test_length_dependent_tables_bit_exact_with_oracle(lib):
    """Dynamic NTK and factor tables (with and without the short table) equal the
    oracle's bit for bit across lengths below, at and above the training length."""
    rng = np.random.default_rng(5)
    for D in (64, 128):
        lam = rng.uniform(1.0, 16.0, D // 2)
        lam_s = rng.uniform(1.0, 1.5, D // 2)
        for seq in (1, 4095, 4096, 4097, 20000, 131072, 1 << 20):
            for mode, kw in (("dynamic_ntk", {}), ("factors", dict(factors=lam)),
                             ("factors", dict(factors=lam, factors_short=lam_s))):
                ref, ref_ms, flags = oracle.rope_table(mode, D, 5e5, 1.0, 4096, 1.0, 32.0,
                                                       seq_len=seq, **kw)
                got, ms = lcx.rope_table(lcx.RopeParams(mode, D, base=5e5,
                                                        original_max_pos=4096, seq_len=seq,
                                                        **kw))
                ok = flags[:-1] == 0
                np.testing.assert_array_equal(got.view(np.uint32)[ok], ref.view(np.uint32)[ok])
                assert ms == ref_ms == 1.0


@pytest.mark.parametrize("bad", [
    dict(head_dim=63), dict(head_dim=0), dict(head_dim=1024), dict(mode="plain", base=1.0),
    dict(mode="pi", scale=0.0), dict(mode="yarn", alpha=32.0, beta=1.0),
    dict(mode="yarn", original_max_pos=0), dict(mode="ntk", head_dim=2),
    dict(mode="yarn", scale=float("nan")),
    dict(mode="factors", seq_len=10),
    dict(mode="factors", seq_len=10, factors=[1.0] * 63 + [0.0]),
    dict(mode="factors", seq_len=10, factors=[1.0] * 64, factors_short=[float("inf")] * 64),
    dict(mode="dynamic_ntk", seq_len=0),
    dict(mode="dynamic_ntk", seq_len=10, original_max_pos=0),
    dict(mode="plain", seq_len=-1),
])
def test_rope_table_rejects_bad_params(lib, bad):
    p = dict(mode="yarn", head_dim=128, scale=4.0, original_max_pos=4096)
    p.update(bad)
    with pytest.raises(lcx.LcxError) as e:
        lcx.rope_table(lcx.RopeParams(**p))
    assert e.value.status == lcx.LCX_ERR_INVALID_ARG


def _apply(lib, params, x, y, dtype, B, H, L, xs, ys=None, pos=0):
    xs_c = (ctypes.c_int64 * 4)(*xs)
    ys_c = (ctypes.c_int64 * 4)(*ys) if ys is not None else None
    p = params._c()
    return lib.lcx_apply_rope(ctypes.byref(p), ctypes.c_void_p(x), ctypes.c_void_p(y), dtype,
                              B, H, L, xs_c, ys_c, pos, None)


def test_apply_rope_validation_without_device(lib):
    """Malformed calls return a status before touching the GPU (pointers are fake
    and never dereferenced)."""
    P = _params("plain", 128)
    fake, fake2 = 0x100000, 0x200000
    cs = [32 * 8 * 128, 8 * 128, 128, 1]
    assert _apply(lib, P, fake, fake2, 7, 1, 32, 8, cs) == lcx.LCX_ERR_INVALID_ARG      # dtype
    assert _apply(lib, P, fake, fake2, 0, -1, 32, 8, cs) == lcx.LCX_ERR_INVALID_ARG     # size
    assert _apply(lib, P, 0, fake2, 0, 1, 32, 8, cs) == lcx.LCX_ERR_INVALID_ARG         # NULL
    assert _apply(lib, P, fake, fake2, 0, 1, 32, 8, cs, pos=-1) == lcx.LCX_ERR_INVALID_ARG
    assert _apply(lib, P, fake + 2, fake2, 0, 1, 32, 8, cs) == lcx.LCX_ERR_UNSUPPORTED  # align
    assert _apply(lib, P, fake, fake2, 0, 1, 32, 8, [cs[0], cs[1], 130, 1]) == \
        lcx.LCX_ERR_UNSUPPORTED                                                          # stride
    assert _apply(lib, P, fake, fake2, 0, 1, 32, 8, [cs[0], cs[1], cs[2], 2]) == \
        lcx.LCX_ERR_UNSUPPORTED                                                          # inner
    assert _apply(lib, _params("plain", 72), fake, fake2, 0, 1, 32, 8,
                  [32 * 8 * 72, 8 * 72, 72, 1]) == lcx.LCX_ERR_UNSUPPORTED               # D%16
    assert _apply(lib, P, fake, fake, 0, 1, 32, 8, cs, [cs[0], cs[1], 256, 1]) == \
        lcx.LCX_ERR_INVALID_ARG                                                          # in place
    # empty tensors are a no-op, even with NULL pointers
    assert _apply(lib, P, 0, 0, 0, 0, 32, 8, cs) == lcx.LCX_OK
    assert _apply(lib, P, 0, 0, 0, 1, 32, 0, cs) == lcx.LCX_OK
    assert lib.lcx_last_error().decode() == ""


def _attn_args(**kw):
    a = lcx._AttnArgs()
    a.q, a.k, a.v, a.o = 0x100000, 0x200000, 0x300000, 0x400000
    a.dtype, a.causal = 0, 1
    a.B, a.Hq, a.Hkv, a.L, a.D = 1, 8, 2, 256, 128
    st_q = [8 * 256 * 128, 256 * 128, 128, 1]
    st_kv = [2 * 256 * 128, 256 * 128, 128, 1]
    a.q_strides = (ctypes.c_int64 * 4)(*st_q)
    a.o_strides = (ctypes.c_int64 * 4)(*st_q)
    a.k_strides = (ctypes.c_int64 * 4)(*st_kv)
    a.v_strides = (ctypes.c_int64 * 4)(*st_kv)
    a.rope = _params("yarn", 128, scale=4.0, original_max_pos=64)._c()
    for k_, v_ in kw.items():
        if k_ == "rope":
            a.rope = v_._c()
        elif k_.endswith("strides"):
            setattr(a, k_, (ctypes.c_int64 * 4)(*v_))
        else:
            setattr(a, k_, v_)
    return a


@pytest.mark.parametrize("kw,expect", [
    (dict(Hkv=3), lcx.LCX_ERR_INVALID_ARG),
    (dict(D=96, rope=_params("plain", 96)), lcx.LCX_ERR_UNSUPPORTED),
    (dict(rope=_params("plain", 130)), lcx.LCX_ERR_INVALID_ARG),     # rotated dims > D
    (dict(dtype=5), lcx.LCX_ERR_INVALID_ARG),
    (dict(causal=2), lcx.LCX_ERR_INVALID_ARG),
    (dict(window=-1), lcx.LCX_ERR_INVALID_ARG),
    (dict(causal=0, window=16), lcx.LCX_ERR_UNSUPPORTED),
    (dict(flags=8), lcx.LCX_ERR_INVALID_ARG),
    (dict(softmax_scale=float("inf")), lcx.LCX_ERR_INVALID_ARG),
    (dict(q=0x100002), lcx.LCX_ERR_UNSUPPORTED),
    (dict(k=0), lcx.LCX_ERR_INVALID_ARG),
    (dict(q_strides=[8 * 256 * 128, 256 * 128, 132, 1]), lcx.LCX_ERR_UNSUPPORTED),
    (dict(v_strides=[2 * 256 * 128, 256 * 128, 128, 2]), lcx.LCX_ERR_UNSUPPORTED),
    (dict(Hq=0), lcx.LCX_ERR_INVALID_ARG),
    (dict(watchdog_ms=-1), lcx.LCX_ERR_INVALID_ARG),
    (dict(watchdog_ms=60001), lcx.LCX_ERR_INVALID_ARG),
    (dict(dtype=1, flags=0x80000000), lcx.LCX_ERR_UNSUPPORTED),
    (dict(reserved0=1), lcx.LCX_ERR_INVALID_ARG),
    (dict(Lk=-1), lcx.LCX_ERR_INVALID_ARG),
    (dict(q_offset=-1), lcx.LCX_ERR_INVALID_ARG),
    (dict(q_offset=1), lcx.LCX_ERR_INVALID_ARG),            # causal: q_offset + L > Lk
    (dict(Lk=255), lcx.LCX_ERR_INVALID_ARG),                # causal: L > Lk
    (dict(Lk=1 << 31, q_offset=(1 << 31) - 256), lcx.LCX_ERR_UNSUPPORTED),
    (dict(Dv=-1), lcx.LCX_ERR_INVALID_ARG),
    (dict(Dv=64), lcx.LCX_ERR_UNSUPPORTED),                           # (128, 64, 128)
    (dict(rope=_params("plain", 256)), lcx.LCX_ERR_INVALID_ARG),      # rotated > D
    (dict(rope=_params("plain", 32)), lcx.LCX_ERR_UNSUPPORTED),       # (128, 128, 32)
    (dict(rope=_params("plain", 64), dtype=1), lcx.LCX_ERR_UNSUPPORTED),   # partial fp32
    (dict(rope=_params("plain", 64), flags=2), lcx.LCX_ERR_UNSUPPORTED),   # partial split
    (dict(k_rope=0x500000), lcx.LCX_ERR_INVALID_ARG),                 # k_rope, full rotary
    (dict(D=192, rope=_params("plain", 192)), lcx.LCX_ERR_UNSUPPORTED),
    (dict(k_rot=0x500008, k_rot_bytes=1 << 30), lcx.LCX_ERR_UNSUPPORTED),  # misaligned
    (dict(k_rot=0x500000, k_rot_bytes=1000), lcx.LCX_ERR_INVALID_ARG),      # too small
    # split QK^T with bf16: the keys' fp16 parts, their cross parts and V in fp16
    # (three times the keys' 131072 bytes); twice is too small
    (dict(k_rot=0x500000, k_rot_bytes=2 * 131072, flags=2), lcx.LCX_ERR_INVALID_ARG),
    (dict(D=192, Dv=128, rope=_params("plain", 64), k_rope=0x500008,
          k_rope_strides=[256 * 64, 256 * 64, 64, 1]), lcx.LCX_ERR_UNSUPPORTED),  # misaligned
    # the shared rotary key rotated once: k_rot must hold [B, 1, Lk, 64]
    (dict(D=192, Dv=128, rope=_params("plain", 64), k_rope=0x500000,
          k_rope_strides=[256 * 64, 256 * 64, 64, 1], k_rot=0x600000, k_rot_bytes=1000),
     lcx.LCX_ERR_INVALID_ARG),
])
def test_attn_validation_without_device(lib, kw, expect):
    a = _attn_args(**kw)
    assert lib.lcx_attn_fwd(ctypes.byref(a), None) == expect
    assert lib.lcx_last_error().decode()


@pytest.mark.parametrize("splits,ws,nbytes", [
    (0, 0x10000000, 1 << 30),        # num_splits out of range
    (257, 0x10000000, 1 << 30),
    (4, 0, 1 << 30),                 # NULL workspace
    (4, 0x10000010, 1 << 30),        # not 256-byte aligned
    (4, 0x10000000, 1000),           # too small
])
def test_attn_split_validation_without_device(lib, splits, ws, nbytes):
    """fp32 operands (no tensor maps are built), so every case stops at the
    split arguments, before any device work."""
    a = _attn_args(dtype=1, q_strides=[8 * 256 * 128, 256 * 128, 128, 1],
                   o_strides=[8 * 256 * 128, 256 * 128, 128, 1])
    assert lib.lcx_attn_fwd_split(ctypes.byref(a), splits, ws, nbytes, None) == \
        lcx.LCX_ERR_INVALID_ARG
    assert lib.lcx_last_error().decode()


def test_split_workspace_bytes(lib):
    f = lib.lcx_attn_split_workspace_bytes
    assert f(1, 32, 1, 128, 1) == 0
    # room for two partial results per split (head-packed launches write one
    # per query tile): [2 S, rows, D] fp32 o then [2 S, rows] fp32 lse, each
    # rounded up to 256 bytes
    assert f(1, 32, 1, 128, 16) == 2 * 16 * 32 * 128 * 4 + 2 * 16 * 32 * 4
    assert f(2, 3, 5, 64, 3) == -(-(6 * 30 * 64 * 4) // 256) * 256 + 768
    for bad in ((1, 32, 1, 96, 4), (1, 32, 1, 128, 0), (1, 32, 1, 128, 257), (-1, 1, 1, 64, 2),
                (1 << 20, 65536, 1 << 30, 128, 2)):
        assert f(*bad) == -1


def test_merge_validation_without_device(lib):
    st = (ctypes.c_int64 * 4)(4 * 8 * 128, 8 * 128, 128, 1)
    m = lib.lcx_attn_merge
    F = 0x10000000
    assert m(F, F, 0, 1, 4, 8, 128, F, 0, st, None, None) == lcx.LCX_ERR_INVALID_ARG
    assert m(F, F, 2, 1, 4, 8, 96, F, 0, st, None, None) == lcx.LCX_ERR_UNSUPPORTED
    assert m(F, F, 2, 1, 4, 8, 128, F, 7, st, None, None) == lcx.LCX_ERR_INVALID_ARG
    assert m(0, F, 2, 1, 4, 8, 128, F, 0, st, None, None) == lcx.LCX_ERR_INVALID_ARG
    assert m(F + 4, F, 2, 1, 4, 8, 128, F, 0, st, None, None) == lcx.LCX_ERR_UNSUPPORTED
    bad = (ctypes.c_int64 * 4)(4 * 8 * 128, 8 * 128, 132, 1)
    assert m(F, F, 2, 1, 4, 8, 128, F, 0, bad, None, None) == lcx.LCX_ERR_UNSUPPORTED
    assert m(0, 0, 2, 0, 4, 8, 128, 0, 0, st, None, None) == lcx.LCX_OK   # empty: no-op


def test_attn_empty_is_noop(lib):
    a = _attn_args(L=0, q=0, k=0, v=0, o=0)
    assert lib.lcx_attn_fwd(ctypes.byref(a), None) == lcx.LCX_OK
    a = _attn_args(B=0)
    assert lib.lcx_attn_fwd(ctypes.byref(a), None) == lcx.LCX_OK
    assert lib.lcx_attn_fwd(None, None) == lcx.LCX_ERR_INVALID_ARG


def test_hf_config_mapping():
    r = lcx.RopeParams.from_hf({"type": "yarn", "factor": 16.0,
                                "original_max_position_embeddings": 8192,
                                "rope_theta": 500000.0}, head_dim=128)
    assert (r.mode, r.scale, r.original_max_pos, r.base) == ("yarn", 16.0, 8192, 500000.0)
    assert lcx.RopeParams.from_hf({"rope_type": "linear", "factor": 4.0}, 64).mode == "pi"


def test_product_path_does_not_touch_the_oracle():
    """The package and its C sources never import, link or name the oracle."""
    pkg = os.path.join(ROOT, "ntk_rope_flashattn_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".cpp", ".h")):
                txt = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert "oracle" not in txt and "orc_" not in txt, f
