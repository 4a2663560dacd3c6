"""The Python binding has no CPU path: without a CUDA device or the built
library it fails loudly instead of computing anything on the host."""
import pytest
import torch

import ntk_rope_flashattn_b200 as lcx


def test_missing_library_raises(monkeypatch, tmp_path):
    monkeypatch.setattr(lcx, "_lib", None)
    with pytest.raises(RuntimeError, match="not found"):
        lcx.load(str(tmp_path / "liblcx.so"))


def _qkv(dtype=torch.bfloat16):
    q = torch.zeros((1, 2, 16, 128), dtype=dtype)
    k = torch.zeros((1, 1, 16, 128), dtype=dtype)
    return q, k, k.clone()


def test_host_tensors_are_refused():
    q, k, v = _qkv()
    rope = lcx.RopeParams("yarn", 128, scale=4.0)
    with pytest.raises(ValueError, match="CUDA"):
        lcx.attn_fwd(q, k, v, rope)
    with pytest.raises(ValueError, match="CUDA"):
        lcx.attn_fwd(q, k, v, rope, num_splits=4)
    with pytest.raises(ValueError, match="CUDA"):
        lcx.apply_rope(q, rope)


def test_host_buffers_are_refused():
    """Every tensor argument is checked, not only q, k and v: a host buffer
    anywhere is refused before the library sees a pointer.  (No CUDA device
    here, so the check is exercised with host q/k/v and every entry point.)"""
    q, k, v = _qkv()
    rope = lcx.RopeParams("plain", 128)
    with pytest.raises(ValueError, match="CUDA"):
        lcx.attn_fwd_split_static(q, k, v, rope, num_splits=2)
    o_parts = torch.zeros((2, 1, 2, 16, 128))
    with pytest.raises(ValueError, match="CUDA"):
        lcx.attn_merge(o_parts, torch.zeros((2, 1, 2, 16)))
    with pytest.raises(ValueError, match="CUDA"):
        lcx._same_device(torch.zeros(1), out=torch.zeros(1))

