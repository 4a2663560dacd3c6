"""GPU parity of decoupled RoPE ("Long Context: RoPE / YaRN / NTK / MLA", 9.5,
9.7 and A.1) against the fp64 oracle: q = [q_C ; q_R], k^(h) = [k_C^(h) ; k_R]
with one rotary key k_R shared by all heads, only the d_R-dim parts rotated
(mscale on them), scores scaled by 1/sqrt(d_C + d_R), values of their own head
dim.  Shapes: DeepSeek-V2's (d_C 128, d_R 64, d_v 128) and d_C = d_R = 64.
Tolerances are those of the prefill tests.
"""
import numpy as np
import pytest
import torch

import ntk_rope_flashattn_b200 as lcx
import oracle
from test_gpu_attn import compare

pytestmark = pytest.mark.gpu


def mla_inputs(B, Hq, Hkv, L, Dc, Dr, Dv, seed=0):
    g = torch.Generator(device="cuda").manual_seed(seed)
    q = torch.randn((B, Hq, L, Dc + Dr), generator=g, device="cuda").bfloat16()
    kc = torch.randn((B, Hkv, L, Dc), generator=g, device="cuda").bfloat16()
    kr = torch.randn((B, 1, L, Dr), generator=g, device="cuda").bfloat16()
    v = torch.randn((B, Hkv, L, Dv), generator=g, device="cuda").bfloat16()
    return q, kc, kr, v


def oracle_mla(q, kc, kr, v, rope, q_offset=0, window=0, sinks=0):
    B, Hq, L, Dq = q.shape
    Lk = kc.shape[2]
    table, ms, _ = oracle.rope_table(rope.mode, rope.head_dim, rope.base, rope.scale,
                                     rope.original_max_pos, rope.alpha, rope.beta,
                                     seq_len=Lk)
    bb, hh, ii = np.meshgrid(np.arange(B), np.arange(Hq), np.arange(L), indexing="ij")
    o, lse = oracle.attn_rows_mla(q.float().cpu().numpy().reshape(-1, Dq), bb.ravel(),
                                  hh.ravel(), ii.ravel() + q_offset, kc.float().cpu().numpy(),
                                  kr[:, 0].float().cpu().numpy(), v.float().cpu().numpy(), Hq,
                                  table, ms, rope.pairing, 0, True, window, sinks)
    return o.reshape(B, Hq, L, -1), lse.reshape(B, Hq, L)


def run(q, k, v, rope, **kw):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = lcx.attn_fwd(q, k, v, rope, return_lse=True, status=status, **kw)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return o, lse


def check(o, lse, ref):
    return compare(o.float().cpu().numpy(), lse.cpu().numpy(), ref[0], ref[1])


YARN = dict(mode="yarn", scale=8.0, original_max_pos=128)


@pytest.mark.parametrize("Dc,Hq,Hkv,L,pairing,window,sinks", [
    (128, 4, 4, 700, "half", 0, 0),            # DeepSeek-V2 head shape, MHA
    (128, 8, 2, 333, "half", 150, 4),          # GQA, window + sinks
    (128, 2, 2, 257, "interleaved", 0, 0),
    (64, 4, 4, 520, "half", 0, 0),             # d_C = d_R = 64
    (64, 4, 2, 300, "interleaved", 100, 2),
    (128, 6, 2, 600, "half", 200, 4),          # G = 3: query-block pairs of one head
])
def test_mla_shared_rope_key(Dc, Hq, Hkv, L, pairing, window, sinks):
    Dr, Dv = 64, 128
    q, kc, kr, v = mla_inputs(1, Hq, Hkv, L, Dc, Dr, Dv, seed=Dc + L)
    rope = lcx.RopeParams(head_dim=Dr, pairing=pairing, **YARN)
    o, lse = run(q, kc, v, rope, k_rope=kr, window=window, sinks=sinks)
    assert o.shape == (1, Hq, L, Dv)
    check(o, lse, oracle_mla(q, kc, kr, v, rope, 0, window, sinks))


@pytest.mark.parametrize("Dc", [128, 64])
def test_mla_per_head_keys_equal_shared(Dc):
    """The rotary part may also sit in every head's own key (k = [k_C ; k_R]
    materialised per head): same result as the shared k_rope."""
    Dr, Dv, Hq, L = 64, 128, 4, 400
    q, kc, kr, v = mla_inputs(2, Hq, Hq, L, Dc, Dr, Dv, seed=5)
    rope = lcx.RopeParams(head_dim=Dr, **YARN)
    k_full = torch.cat([kc, kr.expand(-1, Hq, -1, -1)], dim=-1).contiguous()
    o_full, lse_full = run(q, k_full, v, rope)
    ref = oracle_mla(q, kc, kr, v, rope)
    check(o_full, lse_full, ref)
    o_sh, _ = run(q, kc, v, rope, k_rope=kr)
    assert (o_full.float() - o_sh.float()).abs().max().item() <= 2e-2


def test_mla_decode_split_kv():
    """Decode of 2 new tokens against a 3000-entry cache, 6 key splits, the
    partial outputs in the value head dim."""
    Dc, Dr, Dv, H, Lk = 128, 64, 128, 4, 3000
    q_all, kc, kr, v = mla_inputs(1, H, H, Lk, Dc, Dr, Dv, seed=9)
    q = q_all[:, :, -2:]
    rope = lcx.RopeParams(head_dim=Dr, **YARN)
    o, lse = run(q, kc, v, rope, k_rope=kr, q_offset=Lk - 2, num_splits=6)
    check(o, lse, oracle_mla(q, kc, kr, v, rope, Lk - 2))


def test_mla_prerotated():
    """The rotary slices rotated beforehand by lcx_apply_rope (mscale included):
    q's last d_R columns in place, the shared key out of place."""
    Dc, Dr, Dv, H, L = 128, 64, 128, 4, 300
    q, kc, kr, v = mla_inputs(1, H, H, L, Dc, Dr, Dv, seed=13)
    rope = lcx.RopeParams(head_dim=Dr, **YARN)
    q_rot = q.clone()
    lcx.apply_rope(q_rot[..., Dc:], rope, inplace=True)
    kr_rot = lcx.apply_rope(kr, rope)
    o, lse = run(q_rot, kc, v, rope, k_rope=kr_rot, prerotated=True)
    ref = oracle_mla(q, kc, kr, v, rope)
    check(o, lse, ref)
    o2, lse2 = run(q, kc, v, rope, k_rope=kr_rot, k_prerotated=True)
    check(o2, lse2, ref)


@pytest.mark.parametrize("Dc,Hq,Hkv,L,pairing,window,sinks", [
    (128, 4, 4, 700, "half", 0, 0),            # MHA: query-block pairs
    (128, 8, 2, 333, "half", 150, 4),          # GQA, window + sinks
    (64, 4, 2, 300, "interleaved", 100, 2),
])
def test_mla_rotate_k_once(Dc, Hq, Hkv, L, pairing, window, sinks):
    """The shared rotary key rotated once into k_rot by the rotate pass, the
    kernel reading it from there: the oracle's result, and k_rot equal to
    lcx_apply_rope of the shared key."""
    Dr, Dv = 64, 128
    q, kc, kr, v = mla_inputs(1, Hq, Hkv, L, Dc, Dr, Dv, seed=Dc + L + 1)
    rope = lcx.RopeParams(head_dim=Dr, pairing=pairing, **YARN)
    k_rot = torch.empty_like(kr)
    o, lse = run(q, kc, v, rope, k_rope=kr, window=window, sinks=sinks, k_rot=k_rot)
    check(o, lse, oracle_mla(q, kc, kr, v, rope, 0, window, sinks))
    assert torch.equal(k_rot, lcx.apply_rope(kr, rope))
