"""lcx_attn_fwd_split_static: split-KV attention whose partial results live in
the library's static device scratch (LCX_STATIC_SCRATCH_BYTES per device), so
the call allocates nothing.  Two calls in a row must give exactly what two
calls of lcx_attn_fwd_split with a caller workspace give (same kernels, same
arithmetic), and requests beyond the scratch are refused before device work.

This file is collected last so that it also runs after every other test has
used the library on the device.
"""
import ctypes

import pytest
import torch

import ntk_rope_flashattn_b200 as lcx
from workloads import Workload, make_inputs

W = Workload("static_scratch", B=2, Hq=8, Hkv=2, L=3000, D=128, dtype="bf16", mode="yarn",
             scale=8.0, original_max_pos=256, window=1200, sinks=4)
SCRATCH = 32 * 1024 * 1024
# the first static call: more rows and splits than any checked call, so the
# partial results it leaves cover everything a checked call reads
POISON_L, POISON_SPLITS = 200, 8


def _rope(w):
    return lcx.RopeParams(w.mode, w.D, w.base, w.scale, w.original_max_pos, w.alpha, w.beta)


def _args(**kw):
    a = lcx._AttnArgs()
    a.q, a.k, a.v, a.o = 0x100000, 0x200000, 0x300000, 0x400000
    a.dtype, a.causal = 0, 1
    a.B, a.Hq, a.Hkv, a.L, a.D = 1, 8, 2, 256, 128
    a.q_strides = (ctypes.c_int64 * 4)(8 * 256 * 128, 256 * 128, 128, 1)
    a.o_strides = (ctypes.c_int64 * 4)(8 * 256 * 128, 256 * 128, 128, 1)
    a.k_strides = (ctypes.c_int64 * 4)(2 * 256 * 128, 256 * 128, 128, 1)
    a.v_strides = (ctypes.c_int64 * 4)(2 * 256 * 128, 256 * 128, 128, 1)
    a.rope = lcx.RopeParams("plain", 128)._c()
    for k_, v_ in kw.items():
        setattr(a, k_, v_)
    return a


def test_static_scratch_refuses_before_device_work():
    """Oversize and malformed requests fail on the host (fake pointers: nothing
    may reach the device)."""
    lib = lcx.load()
    a = _args()
    need = lib.lcx_attn_split_workspace_bytes(1, 8, 256, 128, 256)
    assert need > SCRATCH
    assert lib.lcx_attn_fwd_split_static(ctypes.byref(a), 256, None) == lcx.LCX_ERR_UNSUPPORTED
    assert "static" in lib.lcx_last_error().decode()
    assert lib.lcx_attn_fwd_split_static(ctypes.byref(a), 0, None) == lcx.LCX_ERR_INVALID_ARG
    assert lib.lcx_attn_fwd_split_static(ctypes.byref(a), 257, None) == lcx.LCX_ERR_INVALID_ARG
    assert lib.lcx_attn_fwd_split_static(None, 4, None) == lcx.LCX_ERR_INVALID_ARG


@pytest.mark.gpu
@pytest.mark.parametrize("L,splits", [(1, 8), (4, 16), (1, 1), (200, 3)])
def test_static_scratch_equals_workspace_entry(L, splits):
    """Two calls in a row through each entry point: bit-identical o and lse, and
    the static entry allocates no device memory, although an earlier static
    call on other inputs left different partial results in the scratch."""
    q_all, k, v = make_inputs(W, device="cuda")
    q = q_all[:, :, W.L - L:]
    rope = _rope(W)
    kw = dict(window=W.window, sinks=W.sinks, q_offset=W.L - L)
    assert lcx.split_workspace_bytes(W.B, W.Hq, L, W.D, splits) <= SCRATCH
    assert L <= POISON_L and lcx.split_workspace_bytes(W.B, W.Hq, POISON_L, W.D,
                                                       POISON_SPLITS) <= SCRATCH
    ref = [lcx.attn_fwd(q, k, v, rope, num_splits=splits, return_lse=True, **kw)
           for _ in range(2)]
    outs = [(torch.empty_like(q), torch.empty((W.B, W.Hq, L), dtype=torch.float32,
                                              device="cuda")) for _ in range(2)]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    # The first call in a context loads the scratch array (with lazy module
    # loading the CUDA runtime materialises it then); the calls after it are
    # the ones that must allocate nothing.  That first call runs on OTHER
    # inputs (another seed) with more rows and splits, so every byte of the
    # scratch the checked calls read first holds a different, stale value: a
    # partial row the checked call failed to write would show up below.
    q2_all, k2, v2 = make_inputs(W, device="cuda", seed=7)
    lp = POISON_L
    lcx.attn_fwd_split_static(q2_all[:, :, W.L - lp:], k2, v2, rope, POISON_SPLITS,
                              window=W.window, sinks=W.sinks, q_offset=W.L - lp)
    torch.cuda.synchronize()
    allocated, free = torch.cuda.memory_allocated(), torch.cuda.mem_get_info()[0]
    for o, lse in outs:
        lcx.attn_fwd_split_static(q, k, v, rope, splits, out=o, lse=lse, status=status, **kw)
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated() == allocated
    assert torch.cuda.mem_get_info()[0] == free
    assert int(status.item()) == 0
    for (o, lse), (o_ref, lse_ref) in zip(outs, ref):
        assert torch.equal(o, o_ref)
        assert torch.equal(lse, lse_ref)
