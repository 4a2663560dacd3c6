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


@pytest.mark.parametrize("cfg,mode", [
    ({"rope_type": "default"}, "plain"),
    ({"rope_type": "linear", "factor": 4.0}, "pi"),
    ({"type": "ntk", "factor": 4.0}, "ntk"),
    ({"rope_type": "yarn", "factor": 16.0, "original_max_position_embeddings": 8192,
      "beta_slow": 1.0, "beta_fast": 32.0}, "yarn"),
    ({"rope_type": "dynamic", "factor": 2.0, "original_max_position_embeddings": 8192}, "dynamic_ntk"),
])
def test_from_hf_maps_rope_types(cfg, mode):
    """HuggingFace rope types map to the library's modes; "dynamic" is the
    length-dependent NTK base (not a fixed-base NTK table)."""
    r = lcx.RopeParams.from_hf(dict(cfg, rope_theta=500000.0), 128)
    assert r.mode == mode
    assert r.base == 500000.0
    if "original_max_position_embeddings" in cfg:
        assert r.original_max_pos == cfg["original_max_position_embeddings"]
    if "factor" in cfg:
        assert r.scale == cfg["factor"]


def test_from_hf_dynamic_table_depends_on_length():
    """A "dynamic" config gives the plain table up to the training length and
    the NTK-aware base beyond it (lcx_rope_table, host only)."""
    import dataclasses
    r = lcx.RopeParams.from_hf({"rope_type": "dynamic", "max_position_embeddings": 8192}, 128)
    assert r.original_max_pos == 8192
    short, _ = lcx.rope_table(dataclasses.replace(r, seq_len=8192))
    plain, _ = lcx.rope_table(lcx.RopeParams("plain", 128))
    long_, _ = lcx.rope_table(dataclasses.replace(r, seq_len=131072))
    ntk, _ = lcx.rope_table(lcx.RopeParams("ntk", 128, scale=16.0))
    assert (short == plain).all()
    assert (long_ == ntk).all()


def test_from_hf_refuses_unknown_types():
    with pytest.raises(ValueError):
        lcx.RopeParams.from_hf({"rope_type": "longrope"}, 128)
