"""ntk_rope_flashattn_b200 -- RoPE context extension fused into causal attention
prefill on B200 (sm_100a).

Python binding of the C-ABI library ``liblcx.so`` (see ``include/lcx.h``).  It
only marshals arguments: tensors stay PyTorch tensors (device memory and the
current stream come from torch), and every step of the computation runs in the
library's CUDA kernels.  If the library is missing the calls raise; there is no
fallback implementation.

    import torch, ntk_rope_flashattn_b200 as lcx
    rope = lcx.RopeParams("yarn", head_dim=128, scale=16, original_max_pos=8192)
    o = lcx.attn_fwd(q, k, v, rope, causal=True)          # q, k, v: [B, H, L, D]
"""
import ctypes
import os
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblcx.so")

LCX_OK, LCX_ERR_INVALID_ARG, LCX_ERR_UNSUPPORTED, LCX_ERR_CUDA, LCX_ERR_TIMEOUT = range(5)
MODES = {"none": 0, "plain": 1, "pi": 2, "ntk": 3, "yarn": 4, "dynamic_ntk": 5, "factors": 6}
PAIRINGS = {"half": 0, "interleaved": 1}
DTYPES = {"bf16": 0, "f32": 1}
LCX_ATTN_PREROTATED = 1
LCX_ATTN_SPLIT_QK = 2
LCX_ATTN_PREROTATED_K = 4
LCX_ATTN_TEST_STALL = 0x80000000

# Symbols include/lcx.h declares; the library must export every one of them.
EXPORTED = ("lcx_rope_table", "lcx_apply_rope", "lcx_attn_fwd", "lcx_attn_fwd_split",
            "lcx_attn_split_workspace_bytes", "lcx_attn_merge", "lcx_attn_fwd_split_static",
            "lcx_status_string",
            "lcx_last_error", "lcx_version")


class LcxError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__("%s (status %d): %s" % (STATUS_NAMES.get(status, "?"), status, msg))
        self.status = status


STATUS_NAMES = {0: "LCX_OK", 1: "LCX_ERR_INVALID_ARG", 2: "LCX_ERR_UNSUPPORTED",
                3: "LCX_ERR_CUDA", 4: "LCX_ERR_TIMEOUT"}


class _RopeParams(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("pairing", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("base", ctypes.c_double), ("scale", ctypes.c_double),
                ("original_max_pos", ctypes.c_int64), ("alpha", ctypes.c_double),
                ("beta", ctypes.c_double), ("seq_len", ctypes.c_int64),
                ("factors", ctypes.c_void_p), ("factors_short", ctypes.c_void_p)]


class _AttnArgs(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("o", ctypes.c_void_p), ("lse", ctypes.c_void_p),
                ("dev_status", ctypes.c_void_p), ("dtype", ctypes.c_int32),
                ("causal", ctypes.c_int32), ("B", ctypes.c_int64), ("Hq", ctypes.c_int64),
                ("Hkv", ctypes.c_int64), ("L", ctypes.c_int64), ("D", ctypes.c_int64),
                ("q_strides", ctypes.c_int64 * 4), ("k_strides", ctypes.c_int64 * 4),
                ("v_strides", ctypes.c_int64 * 4), ("o_strides", ctypes.c_int64 * 4),
                ("rope", _RopeParams), ("window", ctypes.c_int64), ("sinks", ctypes.c_int64),
                ("softmax_scale", ctypes.c_float), ("flags", ctypes.c_uint32),
                ("watchdog_ms", ctypes.c_int32), ("reserved0", ctypes.c_int32),
                ("Lk", ctypes.c_int64), ("q_offset", ctypes.c_int64), ("Dv", ctypes.c_int64),
                ("k_rope", ctypes.c_void_p), ("k_rope_strides", ctypes.c_int64 * 4),
                ("k_rot", ctypes.c_void_p), ("k_rot_bytes", ctypes.c_int64)]


@dataclass
class RopeParams:
    """RoPE frequency scaling (mirrors ``lcx_rope_params``)."""
    mode: str = "plain"
    head_dim: int = 128
    base: float = 10000.0
    scale: float = 1.0
    original_max_pos: int = 4096
    alpha: float = 1.0
    beta: float = 32.0
    pairing: str = "half"
    seq_len: int = 0              # dynamic_ntk / factors: actual length (0: the call's length)
    factors: object = None        # factors: per-pair lambda_i (head_dim/2 values)
    factors_short: object = None  # factors: optional table for seq_len <= original_max_pos

    @classmethod
    def from_hf(cls, cfg: dict, head_dim: int):
        """From a HuggingFace-style ``rope_scaling`` dict plus ``rope_theta``
        (keys: type/rope_type, factor, original_max_position_embeddings or
        max_position_embeddings, beta_slow -> alpha, beta_fast -> beta,
        rope_theta).  Rope types: default -> plain, linear -> pi, ntk -> ntk,
        yarn -> yarn, dynamic -> dynamic_ntk.  Dynamic NTK here takes its scale
        from the call's context length (s = seq_len / original_max_pos, plain
        RoPE up to the training length), so ``factor`` does not enter it."""
        kind = cfg.get("rope_type", cfg.get("type", "default"))
        mode = {"default": "plain", "linear": "pi", "dynamic": "dynamic_ntk", "ntk": "ntk",
                "yarn": "yarn"}.get(kind, kind)
        if mode not in MODES or mode in ("none", "factors"):
            raise ValueError("rope type %r has no equivalent here" % (kind,))
        lmax = cfg.get("original_max_position_embeddings", cfg.get("max_position_embeddings", 4096))
        return cls(mode=mode, head_dim=head_dim, base=float(cfg.get("rope_theta", 10000.0)),
                   scale=float(cfg.get("factor", 1.0)), original_max_pos=int(lmax),
                   alpha=float(cfg.get("beta_slow", 1.0)), beta=float(cfg.get("beta_fast", 32.0)))

    def _c(self):
        """The C struct; it keeps the factor arrays it points to alive."""
        fl = None if self.factors is None else np.ascontiguousarray(self.factors, np.float64)
        fs = (None if self.factors_short is None
              else np.ascontiguousarray(self.factors_short, np.float64))
        c = _RopeParams(MODES[self.mode], int(self.head_dim), PAIRINGS[self.pairing], 0,
                        float(self.base), float(self.scale), int(self.original_max_pos),
                        float(self.alpha), float(self.beta), int(self.seq_len),
                        None if fl is None else fl.ctypes.data,
                        None if fs is None else fs.ctypes.data)
        c._keep = (fl, fs)
        return c


_lib = None


def load(path: str = LIB_PATH):
    """Load liblcx.so (built by ``python -m ntk_rope_flashattn_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError("liblcx.so not found at %s: build it with "
                           "`python -m ntk_rope_flashattn_b200.build`" % path)
    lib = ctypes.CDLL(path)
    lib.lcx_rope_table.argtypes = [ctypes.POINTER(_RopeParams), ctypes.POINTER(ctypes.c_float),
                                   ctypes.POINTER(ctypes.c_float)]
    lib.lcx_rope_table.restype = ctypes.c_int
    lib.lcx_apply_rope.argtypes = [ctypes.POINTER(_RopeParams), ctypes.c_void_p, ctypes.c_void_p,
                                   ctypes.c_int32, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                   ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int64),
                                   ctypes.c_int64, ctypes.c_void_p]
    lib.lcx_apply_rope.restype = ctypes.c_int
    lib.lcx_attn_fwd.argtypes = [ctypes.POINTER(_AttnArgs), ctypes.c_void_p]
    lib.lcx_attn_fwd.restype = ctypes.c_int
    lib.lcx_attn_fwd_split.argtypes = [ctypes.POINTER(_AttnArgs), ctypes.c_int32, ctypes.c_void_p,
                                       ctypes.c_int64, ctypes.c_void_p]
    lib.lcx_attn_fwd_split.restype = ctypes.c_int
    lib.lcx_attn_fwd_split_static.argtypes = [ctypes.POINTER(_AttnArgs), ctypes.c_int32,
                                              ctypes.c_void_p]
    lib.lcx_attn_fwd_split_static.restype = ctypes.c_int
    lib.lcx_attn_split_workspace_bytes.argtypes = [ctypes.c_int64] * 4 + [ctypes.c_int32]
    lib.lcx_attn_split_workspace_bytes.restype = ctypes.c_int64
    lib.lcx_attn_merge.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32,
                                   ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                   ctypes.c_void_p, ctypes.c_int32,
                                   ctypes.POINTER(ctypes.c_int64), ctypes.c_void_p,
                                   ctypes.c_void_p]
    lib.lcx_attn_merge.restype = ctypes.c_int
    lib.lcx_status_string.argtypes = [ctypes.c_int]
    lib.lcx_status_string.restype = ctypes.c_char_p
    lib.lcx_last_error.argtypes = []
    lib.lcx_last_error.restype = ctypes.c_char_p
    lib.lcx_version.argtypes = []
    lib.lcx_version.restype = ctypes.c_int32
    _lib = lib
    return lib


def _check(st):
    if st != LCX_OK:
        raise LcxError(st, load().lcx_last_error().decode())


def version() -> int:
    return int(load().lcx_version())


def rope_table(rope: RopeParams):
    """(theta' float32[head_dim/2], mscale float32) from ``lcx_rope_table``."""
    lib = load()
    out = np.zeros(rope.head_dim // 2, dtype=np.float32)
    ms = ctypes.c_float(0.0)
    p = rope._c()
    _check(lib.lcx_rope_table(ctypes.byref(p), out.ctypes.data_as(ctypes.POINTER(ctypes.c_float)),
                              ctypes.byref(ms)))
    return out, np.float32(ms.value)


def _dtype_code(t):
    import torch
    if t.dtype == torch.bfloat16:
        return DTYPES["bf16"]
    if t.dtype == torch.float32:
        return DTYPES["f32"]
    raise TypeError("unsupported dtype %s (bf16 or fp32)" % t.dtype)


def _strides(t):
    return (ctypes.c_int64 * 4)(*[int(s) for s in t.stride()])


def _stream(t):
    import torch
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _same_device(ref, **tensors):
    """Every tensor given (None skipped) must be a CUDA tensor on ref's device:
    the library takes device pointers only, so a host buffer is refused here
    rather than handed to a kernel."""
    for name, t in tensors.items():
        if t is not None and (not t.is_cuda or t.device != ref.device):
            raise ValueError("%s must be a CUDA tensor on %s (got %s)" % (name, ref.device,
                                                                         t.device))


def apply_rope(x, rope: RopeParams, out=None, pos_offset: int = 0, inplace: bool = False):
    """Rotate x [B, H, L, D] (bf16/fp32, CUDA) by positions pos_offset + l."""
    import torch
    if x.dim() != 4 or not x.is_cuda:
        raise ValueError("x must be a 4-D CUDA tensor [B, H, L, D]")
    _same_device(x, out=out)
    y = x if inplace else (out if out is not None else torch.empty_like(x))
    B, H, L, D = x.shape
    if D != rope.head_dim:
        raise ValueError("x head_dim %d != rope.head_dim %d" % (D, rope.head_dim))
    p = rope._c()
    _check(load().lcx_apply_rope(ctypes.byref(p), ctypes.c_void_p(x.data_ptr()),
                                 ctypes.c_void_p(y.data_ptr()), _dtype_code(x), B, H, L,
                                 _strides(x), _strides(y), int(pos_offset), _stream(x)))
    return y


def attn_fwd(q, k, v, rope: RopeParams, causal: bool = True, window: int = 0, sinks: int = 0,
             softmax_scale: float = 0.0, return_lse: bool = False, prerotated: bool = False,
             split_qk: bool = False, out=None, lse=None, status=None, watchdog_ms: int = 0,
             q_offset: int = 0, k_prerotated: bool = False, num_splits: int = 1,
             workspace=None, k_rope=None, rotate_k_once: bool = False, k_rot=None,
             _test_stall: bool = False):
    """Fused RoPE + causal attention (prefill, chunked prefill, decode).

    q [B, Hq, L, D], k/v [B, Hkv, Lk, D] CUDA tensors (bf16 or fp32, last dim
    contiguous).  Query row i sits at position q_offset + i and key j at j
    (prefill: q_offset 0 and Lk = L; decode of L new tokens against a cache of
    Lk keys that already holds them: q_offset = Lk - L).  Returns o [B, Hq, L, D]
    (and lse [B, Hq, L] fp32 if asked).
    ``k_prerotated``: k already holds rotated keys (LCX_ATTN_PREROTATED_K), q is
    rotated on chip; ``prerotated``: both are (LCX_ATTN_PREROTATED).
    ``num_splits`` > 1 runs split-KV (lcx_attn_fwd_split): each query block's
    key tiles are shared among that many CTAs and the partial results merged;
    ``workspace`` (uint8 CUDA tensor) is allocated when not given.
    Decoupled RoPE: ``rope.head_dim`` < D rotates only the last
    rope.head_dim dims of q and k; ``k_rope`` [B, 1, Lk, rope.head_dim] then
    supplies that part of every key once for all heads and k holds the first
    D - rope.head_dim dims.  v / o may have their own head dim (v.shape[-1]).
    ``rotate_k_once`` (or a ``k_rot`` buffer shaped like k, three times that in
    the split-QK^T mode with bf16 keys, or like k_rope with decoupled RoPE): the
    keys (with k_rope: the shared rotary key) are rotated once into that buffer
    by the rotate pass before the kernel, which then reads them pre-rotated
    (split mode: as fp16 parts and 8-bit cross parts, with V in fp16 beside
    them), instead of rotating each
    key tile on chip in every CTA that reads it (ignored where the kernel does
    not rotate keys).
    ``split_qk`` (LCX_ATTN_SPLIT_QK) forms QK^T from an fp16 part and e5m2
    cross parts of the rotated operands, for inputs whose large logits bf16
    rounding would spoil (rotated values must stay inside fp16's range).
    ``status`` (optional int32 CUDA tensor of one element) receives
    LCX_ERR_TIMEOUT if a kernel's bounded wait expired (``watchdog_ms``, 0 =
    2000); o and lse are then undefined, and without ``status`` nothing
    reports it.
    """
    import torch
    for t in (q, k, v):
        if t.dim() != 4 or not t.is_cuda:
            raise ValueError("q, k, v must be 4-D CUDA tensors [B, H, L, D]")
    B, Hq, L, D = q.shape
    Hkv, Lk = k.shape[1], k.shape[2]
    Dv = v.shape[3]
    Dk = D - rope.head_dim if k_rope is not None else D
    if k.shape != (B, Hkv, Lk, Dk) or v.shape != (B, Hkv, Lk, Dv):
        raise ValueError("shape mismatch: q %s k %s v %s" % (q.shape, k.shape, v.shape))
    if k_rope is not None and (k_rope.dim() != 4 or k_rope.shape != (B, 1, Lk, rope.head_dim)):
        raise ValueError("k_rope must be [B, 1, Lk, rope.head_dim], got %s" % (k_rope.shape,))
    if not (q.dtype == k.dtype == v.dtype) or (k_rope is not None and k_rope.dtype != q.dtype):
        raise ValueError("q, k, v (and k_rope) must share a dtype")
    _same_device(q, k=k, v=v, out=out, lse=lse, status=status, workspace=workspace,
                 k_rope=k_rope, k_rot=k_rot)
    o = out if out is not None else torch.empty((B, Hq, L, Dv), dtype=q.dtype, device=q.device)
    if return_lse and lse is None:
        lse = torch.empty((B, Hq, L), dtype=torch.float32, device=q.device)
    a = _AttnArgs()
    a.q, a.k, a.v, a.o = q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr()
    a.lse = lse.data_ptr() if lse is not None else None
    a.dev_status = status.data_ptr() if status is not None else None
    a.dtype = _dtype_code(q)
    a.causal = 1 if causal else 0
    a.B, a.Hq, a.Hkv, a.L, a.D = B, Hq, Hkv, L, D
    a.q_strides, a.k_strides, a.v_strides, a.o_strides = (_strides(q), _strides(k),
                                                          _strides(v), _strides(o))
    rope_c = rope._c()
    a.rope = rope_c
    a.window, a.sinks = int(window), int(sinks)
    a.softmax_scale = float(softmax_scale)
    a.flags = ((LCX_ATTN_PREROTATED if prerotated else 0) | (LCX_ATTN_SPLIT_QK if split_qk else 0)
               | (LCX_ATTN_PREROTATED_K if k_prerotated else 0)
               | (LCX_ATTN_TEST_STALL if _test_stall else 0))
    a.watchdog_ms = int(watchdog_ms)
    a.reserved0 = 0
    a.Lk = Lk
    a.q_offset = int(q_offset)
    a.Dv = Dv
    if rotate_k_once and k_rot is None:
        if k_rope is not None:
            # decoupled RoPE: the pass rotates only the shared rotary key
            k_rot = torch.empty((B, 1, Lk, k_rope.shape[-1]), dtype=k.dtype, device=k.device)
        else:
            # split QK^T with bf16 keys: the pass writes the fp16 parts, then the
            # 8-bit cross parts (2 D bytes per key: as many bytes again), then
            # V in fp16 (as many bytes again)
            parts = 3 if (split_qk and k.dtype == torch.bfloat16) else 1
            k_rot = torch.empty((parts, B, Hkv, Lk, Dk), dtype=k.dtype, device=k.device)
    if k_rot is not None:
        a.k_rot = k_rot.data_ptr()
        a.k_rot_bytes = k_rot.numel() * k_rot.element_size()
    if k_rope is not None:
        a.k_rope = k_rope.data_ptr()
        a.k_rope_strides = _strides(k_rope)
    if num_splits == 1:
        _check(load().lcx_attn_fwd(ctypes.byref(a), _stream(q)))
    else:
        need = split_workspace_bytes(B, Hq, L, Dv, num_splits)
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        _check(load().lcx_attn_fwd_split(ctypes.byref(a), int(num_splits),
                                         ctypes.c_void_p(workspace.data_ptr()),
                                         workspace.numel() * workspace.element_size(),
                                         _stream(q)))
    del rope_c
    return (o, lse) if return_lse else o


def attn_fwd_split_static(q, k, v, rope: RopeParams, num_splits: int, causal: bool = True,
                          window: int = 0, sinks: int = 0, softmax_scale: float = 0.0,
                          q_offset: int = 0, out=None, lse=None, status=None,
                          watchdog_ms: int = 0):
    """Split-KV attention through lcx_attn_fwd_split_static: the partial results
    live in the library's static device scratch (LCX_STATIC_SCRATCH_BYTES per
    CUDA context), so nothing is allocated for them.  Calls on one device must
    not overlap in time (they share the scratch).  q [B, Hq, L, D], k/v
    [B, Hkv, Lk, D]; returns o (and fills ``lse`` when given).  If a bounded
    device wait expires (``watchdog_ms``, 0 = 2000) o and lse are undefined;
    pass ``status`` to learn of it (it receives LCX_ERR_TIMEOUT)."""
    import torch
    B, Hq, L, D = q.shape
    Hkv, Lk = k.shape[1], k.shape[2]
    if k.shape != (B, Hkv, Lk, D) or v.shape != k.shape or not (q.dtype == k.dtype == v.dtype):
        raise ValueError("shape / dtype mismatch: q %s k %s v %s" % (q.shape, k.shape, v.shape))
    if not q.is_cuda:
        raise ValueError("q, k, v must be CUDA tensors")
    _same_device(q, k=k, v=v, out=out, lse=lse, status=status)
    o = out if out is not None else torch.empty_like(q)
    a = _AttnArgs()
    a.q, a.k, a.v, a.o = q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr()
    a.lse = lse.data_ptr() if lse is not None else None
    a.dev_status = status.data_ptr() if status is not None else None
    a.dtype = _dtype_code(q)
    a.causal = 1 if causal else 0
    a.B, a.Hq, a.Hkv, a.L, a.D = B, Hq, Hkv, L, D
    a.q_strides, a.k_strides, a.v_strides, a.o_strides = (_strides(q), _strides(k),
                                                          _strides(v), _strides(o))
    rope_c = rope._c()
    a.rope = rope_c
    a.window, a.sinks = int(window), int(sinks)
    a.softmax_scale = float(softmax_scale)
    a.flags = 0
    a.watchdog_ms = int(watchdog_ms)
    a.reserved0 = 0
    a.Lk = Lk
    a.q_offset = int(q_offset)
    _check(load().lcx_attn_fwd_split_static(ctypes.byref(a), int(num_splits), _stream(q)))
    del rope_c
    return o


def split_workspace_bytes(B, Hq, L, D, num_splits):
    """Bytes of workspace lcx_attn_fwd_split needs (0 for one split): fp32
    partial outputs and LSEs for two partial results per split (head-packed
    launches give each of a split's query tiles every other key tile)."""
    n = int(load().lcx_attn_split_workspace_bytes(B, Hq, L, D, int(num_splits)))
    if n < 0:
        raise ValueError("invalid split-KV sizes")
    return n


def attn_merge(o_parts, lse_parts, out=None, lse=None, dtype=None):
    """Merge partial results over disjoint key sets (lcx_attn_merge).

    o_parts [n, B, Hq, L, D] and lse_parts [n, B, Hq, L] fp32 contiguous CUDA
    tensors -> o [B, Hq, L, D] (bf16 unless ``dtype`` or ``out`` says
    otherwise) and lse [B, Hq, L] fp32.
    """
    import torch
    if not o_parts.is_cuda:
        raise ValueError("o_parts must be a CUDA tensor")
    _same_device(o_parts, lse_parts=lse_parts, out=out, lse=lse)
    if o_parts.dtype != torch.float32 or lse_parts.dtype != torch.float32:
        raise ValueError("partial results must be fp32")
    if not (o_parts.is_contiguous() and lse_parts.is_contiguous()):
        raise ValueError("partial results must be contiguous")
    n, B, Hq, L, D = o_parts.shape
    if lse_parts.shape != (n, B, Hq, L):
        raise ValueError("lse_parts shape %s != %s" % (tuple(lse_parts.shape), (n, B, Hq, L)))
    if out is None:
        out = torch.empty((B, Hq, L, D), dtype=dtype or torch.bfloat16, device=o_parts.device)
    if lse is None:
        lse = torch.empty((B, Hq, L), dtype=torch.float32, device=o_parts.device)
    _check(load().lcx_attn_merge(ctypes.c_void_p(o_parts.data_ptr()),
                                 ctypes.c_void_p(lse_parts.data_ptr()), n, B, Hq, L, D,
                                 ctypes.c_void_p(out.data_ptr()), _dtype_code(out), _strides(out),
                                 ctypes.c_void_p(lse.data_ptr()), _stream(o_parts)))
    return out, lse


def host_pieces(B, Hkv, L, chunks, causal=True, q_offset=0, one_piece=False):
    """The pieces attn_fwd_host cuts a call into: (batch or None, first kv head,
    end kv head, first query row, end query row).  About ``chunks`` pieces of
    whole kv-head groups, one batch entry at a time (one piece covering
    everything when ``one_piece``).  Causal prefill (q_offset 0): the first
    piece starts with about its first quarter of query rows and the last piece
    ends with about its last quarter, cut on 128-row query blocks -- a query
    range [i0, i1) needs only the keys [0, i1), so less input is copied before
    the first kernel and less output after the last, and every query tile
    starts where it does in one call over everything."""
    if one_piece:
        return [(None, 0, Hkv, 0, L)]
    per_b = max(1, min(Hkv, -(-int(chunks) // B)))
    bounds = [round(i * Hkv / per_b) for i in range(per_b + 1)]
    pieces = [(b, g0, g1, 0, L) for b in range(B) for g0, g1 in zip(bounds, bounds[1:])
              if g1 > g0]
    q4 = (L // 4) // 128 * 128
    if causal and not q_offset and q4 >= 128:
        c = (L - q4) // 128 * 128           # start of the last piece's rows
        b0, g00, g01, _, _ = pieces[0]
        head = [(b0, g00, g01, 0, q4), (b0, g00, g01, q4, L)]
        if len(pieces) == 1:
            pieces = head[:1] + [(b0, g00, g01, q4, c), (b0, g00, g01, c, L)]
        else:
            bl, gl0, gl1, _, _ = pieces[-1]
            pieces = head + pieces[1:-1] + [(bl, gl0, gl1, 0, c), (bl, gl0, gl1, c, L)]
    return pieces


def attn_fwd_host(q, k, v, rope: RopeParams, device="cuda", workspace=None, chunks=8, **kw):
    """attn_fwd on HOST tensors [B, H, L, D]: copies q/k/v to the device, runs
    the kernel and copies o back to the host (pinned host memory makes the
    copies asynchronous).

    The work is cut into about ``chunks`` pieces of whole kv-head groups (one
    batch entry at a time), and the pieces are pipelined over three streams:
    while the kernel runs on piece c, the inputs of piece c + 1 travel to the
    device and the output of piece c - 1 travels back.  Each piece is one
    lcx_attn_fwd call on views of the device buffers, so the arithmetic is the
    same as one call over everything.  ``workspace`` (dict) keeps the device
    buffers and streams between calls.  Returns the pinned host o; the current
    stream is ordered after the last copy.
    """
    import torch
    ws = workspace if workspace is not None else {}
    B, Hq, L, D = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    dev = {}
    for name, t in (("q", q), ("k", k), ("v", v)):
        buf = ws.get(name)
        if buf is None or buf.shape != t.shape or buf.dtype != t.dtype:
            buf = torch.empty(t.shape, dtype=t.dtype, device=device)
            ws[name] = buf
        dev[name] = buf
    o_shape = (B, Hq, L, v.shape[3])
    o_dev = ws.get("o")
    if o_dev is None or tuple(o_dev.shape) != o_shape or o_dev.dtype != q.dtype:
        o_dev = torch.empty(o_shape, dtype=q.dtype, device=device)
        ws["o"] = o_dev
    o_host = ws.get("o_host")
    if o_host is None or tuple(o_host.shape) != o_shape or o_host.dtype != q.dtype:
        o_host = torch.empty(o_shape, dtype=q.dtype, pin_memory=True)
        ws["o_host"] = o_host
    pieces = host_pieces(B, Hkv, L, chunks, causal=kw.get("causal", True),
                         q_offset=kw.get("q_offset", 0),
                         one_piece="lse" in kw or bool(kw.get("return_lse")))

    def view(t, b, h0, h1, r0=None, r1=None):
        t = t[:, h0:h1] if b is None else t[b:b + 1, h0:h1]
        return t if r0 is None else t[:, :, r0:r1]

    def copy_rows(dst, src, b, h0, h1, r0, r1):
        # rows [r0, r1) of heads [h0, h1): one copy per contiguous block (a
        # strided host <-> device copy would go through a slow staging path)
        if r0 == 0 and r1 == dst.shape[2] and b is not None:
            view(dst, b, h0, h1).copy_(view(src, b, h0, h1), non_blocking=True)
            return
        for bb in (range(dst.shape[0]) if b is None else (b,)):
            for h in range(h0, h1):
                dst[bb, h, r0:r1].copy_(src[bb, h, r0:r1], non_blocking=True)

    cur = torch.cuda.current_stream(device)
    s_in = ws.setdefault("stream_in", torch.cuda.Stream(device))
    s_out = ws.setdefault("stream_out", torch.cuda.Stream(device))
    s_in.wait_stream(cur)
    s_out.wait_stream(cur)
    arrived = []
    have = {}   # (batch, kv head range) -> key rows already on the device
    with torch.cuda.stream(s_in):
        for b, g0, g1, i0, i1 in pieces:
            copy_rows(dev["q"], q, b, g0 * G, g1 * G, i0, i1)
            # keys and values up to the piece's last query (all of them unless
            # causal), from where the group's earlier pieces stopped
            k1 = i1 if i1 < L else k.shape[2]
            k0 = have.get((b, g0, g1), 0)
            if k1 > k0:
                copy_rows(dev["k"], k, b, g0, g1, k0, k1)
                copy_rows(dev["v"], v, b, g0, g1, k0, k1)
                have[(b, g0, g1)] = k1
            ev = torch.cuda.Event()
            ev.record(s_in)
            arrived.append(ev)
    for (b, g0, g1, i0, i1), ev in zip(pieces, arrived):
        cur.wait_event(ev)
        o_piece = view(o_dev, b, g0 * G, g1 * G, i0, i1)
        pkw = dict(kw)
        if i0 > 0 or i1 < L:
            pkw["q_offset"] = i0
        k1 = i1 if i1 < L else k.shape[2]
        attn_fwd(view(dev["q"], b, g0 * G, g1 * G, i0, i1), view(dev["k"], b, g0, g1, 0, k1),
                 view(dev["v"], b, g0, g1, 0, k1), rope, out=o_piece, **pkw)
        done = torch.cuda.Event()
        done.record(cur)
        s_out.wait_event(done)
        with torch.cuda.stream(s_out):
            copy_rows(o_host, o_dev, b, g0 * G, g1 * G, i0, i1)
    cur.wait_stream(s_out)
    return o_host
