"""GPU parity of lcx_attn_fwd with query position offsets: chunked prefill,
decode against a key cache, a pre-rotated key cache, and the StreamingLLM
decode loop over a cache of un-rotated keys ("Long Context: RoPE / YaRN / NTK /
MLA", section 10.3), all against the fp64 oracle.

Query row i of a call sits at position q_offset + i and key j at position j;
the oracle is given the same positions (row index q_offset + i into the key
arrays).  Tolerances are those of the prefill tests (test_gpu_attn.py).
"""
import numpy as np
import pytest
import torch

import ntk_rope_flashattn_b200 as lcx
import oracle
from test_gpu_attn import compare
from workloads import Workload, make_inputs

pytestmark = pytest.mark.gpu


def oracle_rows(q, k, v, rope, q_offset, causal=True, window=0, sinks=0):
    """Oracle output for every row of q [B, Hq, L, D] at positions q_offset + i
    against k/v [B, Hkv, Lk, D] at positions 0..Lk-1."""
    B, Hq, L, D = q.shape
    table, ms, _ = oracle.rope_table(rope.mode, D, rope.base, rope.scale, rope.original_max_pos,
                                     rope.alpha, rope.beta, seq_len=k.shape[2])
    bb, hh, ii = np.meshgrid(np.arange(B), np.arange(Hq), np.arange(L), indexing="ij")
    o, lse = oracle.attn_rows(q.float().cpu().numpy().reshape(-1, D), bb.ravel(), hh.ravel(),
                              ii.ravel() + q_offset, k.float().cpu().numpy(),
                              v.float().cpu().numpy(), Hq, table, ms, rope.pairing, 0, causal,
                              window, sinks)
    return o.reshape(B, Hq, L, D), lse.reshape(B, Hq, L)


def run(q, k, v, rope, **kw):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = lcx.attn_fwd(q, k, v, rope, return_lse=True, status=status, **kw)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return o, lse


def check(o, lse, ref, bits=8):
    return compare(o.float().cpu().numpy(), lse.cpu().numpy(), ref[0], ref[1], bits)


W0 = Workload("decode", B=1, Hq=4, Hkv=2, L=1000, D=128, dtype="bf16", mode="yarn", scale=8.0,
              original_max_pos=128)


def rope_of(w):
    return lcx.RopeParams(w.mode, w.D, w.base, w.scale, w.original_max_pos, w.alpha, w.beta,
                          w.pairing)


@pytest.mark.parametrize("window,sinks", [(0, 0), (300, 4)])
def test_chunked_prefill(window, sinks):
    """Prefill in three chunks (each chunk's queries against all keys so far)
    equals the oracle, and agrees with the one-call prefill."""
    w = W0
    q, k, v = make_inputs(w, device="cuda")
    rope = rope_of(w)
    full_o, _ = run(q, k, v, rope, window=window, sinks=sinks)
    for a, b in ((0, 300), (300, 701), (701, 1000)):
        qc, kc, vc = q[:, :, a:b], k[:, :, :b], v[:, :, :b]     # strided views
        o, lse = run(qc, kc, vc, rope, window=window, sinks=sinks, q_offset=a)
        check(o, lse, oracle_rows(qc, kc, vc, rope, a, True, window, sinks))
        diff = (o.float() - full_o[:, :, a:b].float()).abs().max().item()
        assert diff <= 4e-2, diff


@pytest.mark.parametrize("name,kw", [
    ("one_token", dict(L=1)),
    ("one_token_G4", dict(L=1, Hq=8, Hkv=2, mode="ntk", scale=4.0)),
    ("four_tokens_window_sinks", dict(L=4, window=100, sinks=4)),
    ("one_token_D64_interleaved", dict(L=1, D=64, pairing="interleaved")),
    ("three_tokens_f32", dict(L=3, dtype="f32", mode="pi", scale=2.0)),
    ("two_tokens_split", dict(L=2, split_qk=True, window=200, sinks=2)),
    ("one_token_B2_MHA", dict(L=1, B=2, Hq=2, Hkv=2)),
])
def test_decode(name, kw):
    """L new queries (the last L positions) against a cache of Lk = 777 keys."""
    Lk = 777
    w = W0.with_(**{k_: v_ for k_, v_ in kw.items() if k_ not in ("L",)}, L=Lk)
    q_all, k, v = make_inputs(w, device="cuda")
    L = kw["L"]
    q = q_all[:, :, Lk - L:]
    rope = rope_of(w)
    o, lse = run(q, k, v, rope, window=w.window, sinks=w.sinks, q_offset=Lk - L,
                 split_qk=w.split_qk)
    check(o, lse, oracle_rows(q, k, v, rope, Lk - L, True, w.window, w.sinks),
          24 if w.dtype == "f32" else 8)


def test_decode_non_causal_offset():
    """Without the causal mask the offset only moves the query rotation."""
    w = W0.with_(L=300)
    q, k, v = make_inputs(w, device="cuda")
    rope = rope_of(w)
    o, lse = run(q[:, :, 100:150], k, v, rope, causal=False, q_offset=100)
    check(o, lse, oracle_rows(q[:, :, 100:150], k, v, rope, 100, False))


def test_prerotated_key_cache():
    """A cache of keys rotated by lcx_apply_rope (mscale included) with the new
    queries rotated on chip at their offsets."""
    w = W0.with_(L=640)
    q, k, v = make_inputs(w, device="cuda")
    rope = rope_of(w)
    k_rot = lcx.apply_rope(k, rope)
    a = 600
    o, lse = run(q[:, :, a:], k_rot, v, rope, q_offset=a, k_prerotated=True, window=256,
                 sinks=4)
    check(o, lse, oracle_rows(q[:, :, a:], k, v, rope, a, True, 256, 4))


def test_streaming_llm_decode_loop():
    """StreamingLLM decode ("Long Context", section 10.3): the cache keeps the S
    first and W most recent tokens with their keys un-rotated; each step the new
    token (position = current cache length) attends to the cache plus itself,
    every cached key re-rotated at its index in the cache, then the cache is
    trimmed back to S + W entries."""
    S, W, prompt, steps = 4, 60, 150, 40
    w = W0.with_(L=prompt + steps)
    q_all, k_all, v_all = make_inputs(w, device="cuda")
    rope = rope_of(w)
    # the prompt's un-rotated keys, trimmed to sinks + recent window
    k_cache = torch.cat([k_all[:, :, :S], k_all[:, :, prompt - W:prompt]], dim=2)
    v_cache = torch.cat([v_all[:, :, :S], v_all[:, :, prompt - W:prompt]], dim=2)
    for t in range(prompt, prompt + steps):
        cur = k_cache.shape[2]
        kc = torch.cat([k_cache, k_all[:, :, t:t + 1]], dim=2)
        vc = torch.cat([v_cache, v_all[:, :, t:t + 1]], dim=2)
        q = q_all[:, :, t:t + 1]
        o, lse = run(q, kc, vc, rope, q_offset=cur)
        check(o, lse, oracle_rows(q, kc, vc, rope, cur))
        k_cache = torch.cat([kc[:, :, :S], kc[:, :, -W:]], dim=2)
        v_cache = torch.cat([vc[:, :, :S], vc[:, :, -W:]], dim=2)
