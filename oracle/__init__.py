"""fp64 CPU oracle for RoPE context extension + causal attention prefill.

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg are the only callers.  The CUDA library never
imports or links anything here, and this package imports nothing from it.

Thin ctypes wrappers around ``liblcx_oracle.so`` (plain C, fp64); see
``lcx_oracle.c`` for the definitions and their sources.
"""
import ctypes

import numpy as np

from . import build as _build

MODES = {"none": 0, "plain": 1, "pi": 2, "ntk": 3, "yarn": 4, "dynamic_ntk": 5, "factors": 6}
PAIRINGS = {"half": 0, "interleaved": 1}

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        i64p = ctypes.POINTER(ctypes.c_int64)
        f32p = ctypes.POINTER(ctypes.c_float)
        f64p = ctypes.POINTER(ctypes.c_double)
        i32p = ctypes.POINTER(ctypes.c_int)
        lib.orc_rope_theta_fp64.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                            ctypes.c_double, ctypes.c_int64, ctypes.c_double,
                                            ctypes.c_double, f64p, f64p]
        lib.orc_rope_table.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                       ctypes.c_double, ctypes.c_int64, ctypes.c_double,
                                       ctypes.c_double, f32p, f32p, f64p, i32p]
        lib.orc_rope_table_ext.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                           ctypes.c_double, ctypes.c_int64, ctypes.c_double,
                                           ctypes.c_double, ctypes.c_int64, f64p, f64p, f32p,
                                           f32p, f64p, i32p]
        lib.orc_rope_theta_ext.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                           ctypes.c_double, ctypes.c_int64, ctypes.c_double,
                                           ctypes.c_double, ctypes.c_int64, f64p, f64p, f64p,
                                           f64p]
        lib.orc_rotate_rows.argtypes = [f32p, f64p, ctypes.c_int64, ctypes.c_int, i64p,
                                        f32p, ctypes.c_float, ctypes.c_int]
        lib.orc_visible.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                    ctypes.c_int, ctypes.c_int64, ctypes.c_int64]
        lib.orc_mask.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int64, ctypes.c_int64,
                                 ctypes.POINTER(ctypes.c_uint8)]
        lib.orc_mask.restype = None
        lib.orc_attn_rows.argtypes = [f32p, i64p, i64p, i64p, ctypes.c_int64, f32p, f32p,
                                      ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                      ctypes.c_int64, ctypes.c_int64, f32p, ctypes.c_float,
                                      ctypes.c_int, ctypes.c_int64, ctypes.c_int,
                                      ctypes.c_int64, ctypes.c_int64, ctypes.c_double,
                                      f64p, f64p, ctypes.c_int]
        lib.orc_attn_rows_keys.argtypes = (lib.orc_attn_rows.argtypes[:19] +
                                           [ctypes.c_int64, ctypes.c_int64] +
                                           lib.orc_attn_rows.argtypes[19:])
        lib.orc_merge.argtypes = [f64p, f64p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                  f64p, f64p]
        lib.orc_attn_rows_mla.argtypes = [f32p, i64p, i64p, i64p, ctypes.c_int64, f32p, f32p,
                                          f32p] + [ctypes.c_int64] * 7 + [
                                          f32p, ctypes.c_float, ctypes.c_int, ctypes.c_int64,
                                          ctypes.c_int, ctypes.c_int64, ctypes.c_int64,
                                          ctypes.c_double, f64p, f64p, ctypes.c_int]
        lib.orc_num_threads.argtypes = [ctypes.c_int]
        _lib = lib
    return _lib


def _ptr(a, ct):
    return a.ctypes.data_as(ctypes.POINTER(ct))


def rope_theta_fp64(mode, D, base=10000.0, scale=1.0, original_max_pos=4096,
                    alpha=1.0, beta=32.0):
    """theta'_i in fp64 (before the fp32 rounding) and mscale in fp64."""
    lib = _load()
    out = np.zeros(D // 2, dtype=np.float64)
    ms = ctypes.c_double(0.0)
    rc = lib.orc_rope_theta_fp64(MODES[mode], D, base, scale, original_max_pos, alpha, beta,
                                 _ptr(out, ctypes.c_double), ctypes.byref(ms))
    if rc:
        raise ValueError("orc_rope_theta_fp64: invalid argument")
    return out, ms.value


def _f64_or_null(a):
    if a is None:
        return None, None
    a = np.ascontiguousarray(a, dtype=np.float64)
    return a, _ptr(a, ctypes.c_double)


def rope_table(mode, D, base=10000.0, scale=1.0, original_max_pos=4096, alpha=1.0, beta=32.0,
               seq_len=0, factors=None, factors_short=None):
    """fp32 table (theta'_i rounded to nearest even), fp32 mscale, midpoint flags.

    flags has D/2 + 1 entries (the last one for mscale); a 1 marks a value whose
    fp32 rounding is too close to a midpoint to be trusted bit for bit.
    seq_len / factors / factors_short are used by the dynamic_ntk and factors modes.
    """
    lib = _load()
    table = np.zeros(D // 2, dtype=np.float32)
    ms = ctypes.c_float(0.0)
    flags = np.zeros(D // 2 + 1, dtype=np.int32)
    fa, fp = _f64_or_null(factors)
    fsa, fsp = _f64_or_null(factors_short)
    rc = lib.orc_rope_table_ext(MODES[mode], D, base, scale, original_max_pos, alpha, beta,
                                int(seq_len), fp, fsp, _ptr(table, ctypes.c_float),
                                ctypes.byref(ms), None, _ptr(flags, ctypes.c_int))
    if rc:
        raise ValueError("orc_rope_table: invalid argument")
    return table, np.float32(ms.value), flags


def rope_theta_ext(mode, D, base=10000.0, scale=1.0, original_max_pos=4096, alpha=1.0,
                   beta=32.0, seq_len=0, factors=None, factors_short=None):
    """fp64 theta'_i and mscale for every mode, including the length-dependent ones."""
    lib = _load()
    out = np.zeros(D // 2, dtype=np.float64)
    ms = ctypes.c_double(0.0)
    fa, fp = _f64_or_null(factors)
    fsa, fsp = _f64_or_null(factors_short)
    rc = lib.orc_rope_theta_ext(MODES[mode], D, base, scale, original_max_pos, alpha, beta,
                                int(seq_len), fp, fsp, _ptr(out, ctypes.c_double),
                                ctypes.byref(ms))
    if rc:
        raise ValueError("orc_rope_theta_ext: invalid argument")
    return out, ms.value


def rotate_rows(x, pos, table, mscale, pairing="half"):
    """Rotate rows x[n, D] (fp32 values) at integer positions pos[n]; fp64 out."""
    lib = _load()
    x = np.ascontiguousarray(x, dtype=np.float32)
    n, D = x.shape
    pos = np.ascontiguousarray(pos, dtype=np.int64)
    assert pos.shape == (n,)
    table = np.ascontiguousarray(table, dtype=np.float32)
    y = np.zeros((n, D), dtype=np.float64)
    rc = lib.orc_rotate_rows(_ptr(x, ctypes.c_float), _ptr(y, ctypes.c_double), n, D,
                             _ptr(pos, ctypes.c_int64), _ptr(table, ctypes.c_float),
                             float(mscale), PAIRINGS[pairing])
    if rc:
        raise ValueError("orc_rotate_rows: invalid argument")
    return y


def visible(i, j, L, causal=True, window=0, sinks=0):
    return bool(_load().orc_visible(i, j, L, int(causal), window, sinks))


def mask(L, causal=True, window=0, sinks=0):
    """[L, L] bool visibility mask (True = key j visible to query i)."""
    m = np.zeros((L, L), dtype=np.uint8)
    _load().orc_mask(L, int(causal), window, sinks, _ptr(m, ctypes.c_uint8))
    return m.astype(bool)


def attn_rows(q_rows, row_b, row_h, row_i, k, v, Hq, table, mscale, pairing="half",
                 pos_offset=0, causal=True, window=0, sinks=0, scale=None, nthreads=0,
                 k_begin=0, k_end=None):
    """Attention output o[n, D] and lse[n] (fp64) for selected query rows.

    q_rows: [n, D] raw (un-rotated) query rows; row_b/row_h/row_i: batch, query
    head and query index of each row; k, v: [B, Hkv, L, D] raw keys / values
    (fp32 arrays holding the exact input values); Hq: number of query heads
    (query head h reads kv head h // (Hq // Hkv)).  k_begin/k_end restrict the
    keys to k_begin <= j < k_end (a partial result for merge()).
    """
    lib = _load()
    q_rows = np.ascontiguousarray(q_rows, dtype=np.float32)
    k = np.ascontiguousarray(k, dtype=np.float32)
    v = np.ascontiguousarray(v, dtype=np.float32)
    row_b = np.ascontiguousarray(row_b, dtype=np.int64)
    row_h = np.ascontiguousarray(row_h, dtype=np.int64)
    row_i = np.ascontiguousarray(row_i, dtype=np.int64)
    return _attn_rows_impl(lib, q_rows, row_b, row_h, row_i, k, v, Hq, table, mscale,
                           pairing, pos_offset, causal, window, sinks, scale, nthreads,
                           k_begin, k_end)


def _attn_rows_impl(lib, q_rows, row_b, row_h, row_i, k, v, Hq, table, mscale, pairing,
                    pos_offset, causal, window, sinks, scale, nthreads, k_begin=0, k_end=None):
    B, Hkv, L, D = k.shape
    if k_end is None:
        k_end = L
    n = q_rows.shape[0]
    assert q_rows.shape == (n, D)
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    table = np.ascontiguousarray(table, dtype=np.float32)
    o = np.zeros((n, D), dtype=np.float64)
    lse = np.zeros(n, dtype=np.float64)
    rc = lib.orc_attn_rows_keys(_ptr(q_rows, ctypes.c_float), _ptr(row_b, ctypes.c_int64),
                                _ptr(row_h, ctypes.c_int64), _ptr(row_i, ctypes.c_int64), n,
                                _ptr(k, ctypes.c_float), _ptr(v, ctypes.c_float),
                                B, Hq, Hkv, L, D, _ptr(table, ctypes.c_float), float(mscale),
                                PAIRINGS[pairing], int(pos_offset), int(causal), int(window),
                                int(sinks), int(k_begin), int(k_end), float(scale),
                                _ptr(o, ctypes.c_double), _ptr(lse, ctypes.c_double),
                                int(nthreads))
    if rc:
        raise ValueError("orc_attn_rows: invalid argument (rc=%d)" % rc)
    return o, lse


def attn_full(q, k, v, table, mscale, pairing="half", pos_offset=0, causal=True,
              window=0, sinks=0, scale=None, nthreads=0):
    """All rows: q [B, Hq, L, D], k/v [B, Hkv, L, D] -> o [B, Hq, L, D], lse [B, Hq, L]."""
    q = np.asarray(q, dtype=np.float32)
    B, Hq, L, D = q.shape
    bb, hh, ii = np.meshgrid(np.arange(B), np.arange(Hq), np.arange(L), indexing="ij")
    o, lse = attn_rows(q.reshape(-1, D), bb.ravel(), hh.ravel(), ii.ravel(), k, v, Hq,
                          table, mscale, pairing, pos_offset, causal, window, sinks, scale,
                          nthreads)
    return o.reshape(B, Hq, L, D), lse.reshape(B, Hq, L)


def num_threads(nthreads=0):
    return int(_load().orc_num_threads(nthreads))


def merge(o_parts, lse_parts):
    """Combine partial results over disjoint key sets: o_parts [n, ..., D] and
    lse_parts [n, ...] (fp64) -> o [..., D], lse [...] (see orc_merge)."""
    o_parts = np.ascontiguousarray(o_parts, dtype=np.float64)
    lse_parts = np.ascontiguousarray(lse_parts, dtype=np.float64)
    n, D = o_parts.shape[0], o_parts.shape[-1]
    lead = lse_parts.shape[1:]
    assert o_parts.shape == (n,) + lead + (D,)
    rows = int(np.prod(lead)) if lead else 1
    o = np.zeros(lead + (D,), dtype=np.float64)
    lse = np.zeros(lead, dtype=np.float64)
    rc = _load().orc_merge(_ptr(o_parts, ctypes.c_double), _ptr(lse_parts, ctypes.c_double),
                           n, rows, D, _ptr(o, ctypes.c_double), _ptr(lse, ctypes.c_double))
    if rc:
        raise ValueError("orc_merge: invalid argument (rc=%d)" % rc)
    return o, lse


def attn_rows_mla(q_rows, row_b, row_h, row_i, kc, kr, v, Hq, table, mscale, pairing="half",
                  pos_offset=0, causal=True, window=0, sinks=0, scale=None, nthreads=0):
    """Decoupled-RoPE attention (see orc_attn_rows_mla) for selected query rows.

    q_rows [n, Dc + Dr]; kc [B, Hkv, L, Dc] (Dc may be 0); kr [B, L, Dr] shared by
    all heads; v [B, Hkv, L, Dv]; table of a Dr-dim RoPE.  Default scale
    1/sqrt(Dc + Dr).  Returns o [n, Dv], lse [n] in fp64.
    """
    q_rows = np.ascontiguousarray(q_rows, dtype=np.float32)
    kc = np.ascontiguousarray(kc, dtype=np.float32)
    kr = np.ascontiguousarray(kr, dtype=np.float32)
    v = np.ascontiguousarray(v, dtype=np.float32)
    B, Hkv, L, Dc = kc.shape
    Dr, Dv = kr.shape[2], v.shape[3]
    assert kr.shape == (B, L, Dr) and v.shape[:3] == (B, Hkv, L)
    n = q_rows.shape[0]
    assert q_rows.shape == (n, Dc + Dr)
    if scale is None:
        scale = 1.0 / np.sqrt(Dc + Dr)
    row_b, row_h, row_i = (np.ascontiguousarray(x, dtype=np.int64) for x in (row_b, row_h, row_i))
    table = np.ascontiguousarray(table, dtype=np.float32)
    o = np.zeros((n, Dv), dtype=np.float64)
    lse = np.zeros(n, dtype=np.float64)
    kc_p = kc if kc.size else np.zeros(1, np.float32)
    rc = _load().orc_attn_rows_mla(_ptr(q_rows, ctypes.c_float), _ptr(row_b, ctypes.c_int64),
                                   _ptr(row_h, ctypes.c_int64), _ptr(row_i, ctypes.c_int64), n,
                                   _ptr(kc_p, ctypes.c_float), _ptr(kr, ctypes.c_float),
                                   _ptr(v, ctypes.c_float), B, Hq, Hkv, L, Dc, Dr, Dv,
                                   _ptr(table, ctypes.c_float), float(mscale), PAIRINGS[pairing],
                                   int(pos_offset), int(causal), int(window), int(sinks),
                                   float(scale), _ptr(o, ctypes.c_double),
                                   _ptr(lse, ctypes.c_double), int(nthreads))
    if rc:
        raise ValueError("orc_attn_rows_mla: invalid argument (rc=%d)" % rc)
    return o, lse
