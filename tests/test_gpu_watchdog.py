"""The attention kernel's bounded waits, exercised without faulting the GPU.

With the LCX_ATTN_TEST_STALL hook the loader issues no copies, so every wait in
the kernel runs out after watchdog_ms: the kernel must end on its own, report
LCX_ERR_TIMEOUT through the status word and leave the context usable.
"""
import time

import pytest
import torch

import ntk_rope_flashattn_b200 as lcx
from workloads import Workload, make_inputs

pytestmark = pytest.mark.gpu


def test_expired_waits_report_timeout_and_context_survives():
    w = Workload("stall", B=1, Hq=4, Hkv=2, L=1024, D=128, dtype="bf16", mode="yarn",
                 scale=4.0, original_max_pos=256)
    q, k, v = make_inputs(w, device="cuda")
    rope = lcx.RopeParams(w.mode, w.D, w.base, w.scale, w.original_max_pos)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    lcx.attn_fwd(q, k, v, rope, status=status, watchdog_ms=50, _test_stall=True)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert int(status.item()) == lcx.LCX_ERR_TIMEOUT
    # 32 work units, each gives up after about 50 ms (later ones skip at once)
    assert elapsed < 10.0
    # the context still works: a normal call afterwards succeeds and is correct
    status.zero_()
    o1 = lcx.attn_fwd(q, k, v, rope, status=status)
    o2 = lcx.attn_fwd(q, k, v, rope)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.equal(o1, o2) and torch.isfinite(o1.float()).all()


def test_decode_kernel_expired_waits_report_timeout():
    """The same for the transposed-score decode kernel (split-KV, one token per
    query head): with no copies issued every CTA gives up after watchdog_ms,
    the status word reads LCX_ERR_TIMEOUT, and decode calls afterwards succeed
    and agree with the unsplit kernel."""
    w = Workload("stall_decode", B=1, Hq=8, Hkv=2, L=2048, D=128, dtype="bf16", mode="yarn",
                 scale=4.0, original_max_pos=256)
    q, k, v = make_inputs(w, device="cuda")
    qd = q[:, :, -1:].contiguous()
    rope = lcx.RopeParams(w.mode, w.D, w.base, w.scale, w.original_max_pos)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    lcx.attn_fwd(qd, k, v, rope, status=status, watchdog_ms=50, _test_stall=True,
                 q_offset=w.L - 1, num_splits=4)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert int(status.item()) == lcx.LCX_ERR_TIMEOUT
    assert elapsed < 10.0
    status.zero_()
    o_split = lcx.attn_fwd(qd, k, v, rope, status=status, q_offset=w.L - 1, num_splits=4)
    o_plain = lcx.attn_fwd(qd, k, v, rope, q_offset=w.L - 1)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.isfinite(o_split.float()).all()
    assert float((o_split.float() - o_plain.float()).abs().max()) <= 2e-2
