"""GPU parity of split-KV attention (lcx_attn_fwd_split) and the (O, LSE) merge
(lcx_attn_merge) against the fp64 oracle ("8.3 长上下文技术", 8.3.4 online
softmax and 8.3.5 step 3: partial results over disjoint key sets combined by
their softmax statistics).

Split-KV must give the unsplit result up to rounding, for any split count
(including more splits than a query block has key tiles, which leaves empty
splits), so every case is checked against the oracle with the prefill
tolerances; the merge kernel is checked against the oracle's merge.
"""
import numpy as np
import pytest
import torch

import ntk_rope_flashattn_b200 as lcx
import oracle
from test_gpu_attn import compare
from test_gpu_decode import W0, oracle_rows, rope_of
from workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


def run_split(q, k, v, rope, num_splits, **kw):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = lcx.attn_fwd(q, k, v, rope, return_lse=True, status=status, num_splits=num_splits,
                          **kw)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return o, lse


@pytest.mark.parametrize("L,Lk,splits,extra", [
    (1, 777, 3, {}),
    (1, 777, 16, {}),                        # more splits than the 7 key tiles
    (4, 5000, 8, dict(window=1000, sinks=4)),
    (1, 4096, 32, dict(Hq=8, Hkv=2)),
    (2, 900, 5, dict(split_qk=True, window=300, sinks=2)),
    (3, 640, 4, dict(dtype="f32", mode="pi", scale=2.0)),
    (1, 500, 7, dict(D=64, pairing="interleaved")),
    (300, 2000, 3, dict(Hq=2, Hkv=2)),       # G = 1, too many rows to pack: query-block pairs
])
def test_splitkv_decode(L, Lk, splits, extra):
    w = W0.with_(**extra, L=Lk)
    q_all, k, v = make_inputs(w, device="cuda")
    q = q_all[:, :, Lk - L:]
    rope = rope_of(w)
    o, lse = run_split(q, k, v, rope, splits, window=w.window, sinks=w.sinks, q_offset=Lk - L,
                       split_qk=w.split_qk)
    ref = oracle_rows(q, k, v, rope, Lk - L, True, w.window, w.sinks)
    compare(o.float().cpu().numpy(), lse.cpu().numpy(), ref[0], ref[1],
            24 if w.dtype == "f32" else 8)


@pytest.mark.parametrize("splits", [2, 5])
def test_splitkv_prefill(splits):
    """Prefill with split keys: causal rows of every length, window and sinks."""
    w = W0.with_(L=700, window=250, sinks=3)
    q, k, v = make_inputs(w, device="cuda")
    rope = rope_of(w)
    o, lse = run_split(q, k, v, rope, splits, window=w.window, sinks=w.sinks)
    ref = oracle_rows(q, k, v, rope, 0, True, w.window, w.sinks)
    compare(o.float().cpu().numpy(), lse.cpu().numpy(), ref[0], ref[1])
    o1, _ = run_split(q, k, v, rope, 1, window=w.window, sinks=w.sinks)
    assert (o.float() - o1.float()).abs().max().item() <= 2e-2


def test_splitkv_deterministic_and_workspace_reuse():
    w = W0.with_(L=3000)
    q_all, k, v = make_inputs(w, device="cuda")
    q = q_all[:, :, -2:]
    rope = rope_of(w)
    ws = torch.empty(lcx.split_workspace_bytes(1, w.Hq, 2, w.D, 6), dtype=torch.uint8,
                     device="cuda")
    a = lcx.attn_fwd(q, k, v, rope, q_offset=2998, num_splits=6, workspace=ws)
    ws.fill_(0xFF)                            # stale contents must not matter
    b = lcx.attn_fwd(q, k, v, rope, q_offset=2998, num_splits=6, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_splitkv_long_cache_sampled():
    """One new token per head against the 131072-key cache of the YaRN s=16
    workload, 16 splits."""
    w = WORKLOADS["yarn_L131072_s16"]
    q_all, k, v = make_inputs(w, device="cuda")
    q = q_all[:, :, -1:].contiguous()
    del q_all
    rope = rope_of(w)
    o, lse = run_split(q, k, v, rope, 16, q_offset=w.L - 1)
    ref = oracle_rows(q, k, v, rope, w.L - 1)
    compare(o.float().cpu().numpy(), lse.cpu().numpy(), ref[0], ref[1])


@pytest.mark.parametrize("D,dtype", [(128, torch.bfloat16), (64, torch.float32)])
def test_merge_matches_oracle(D, dtype):
    n, B, Hq, L = 5, 2, 3, 37
    g = torch.Generator(device="cuda").manual_seed(7)
    o_parts = torch.randn((n, B, Hq, L, D), generator=g, device="cuda")
    lse_parts = 3.0 * torch.randn((n, B, Hq, L), generator=g, device="cuda")
    lse_parts[1, 0, 0, :5] = -float("inf")        # empty parts
    lse_parts[:, 1, 2, 7] = -float("inf")         # a row with no key at all
    base = torch.empty((B, L, Hq, D + 8), dtype=dtype, device="cuda")
    out = base[..., :D].permute(0, 2, 1, 3)      # strided output [B, Hq, L, D]
    o, lse = lcx.attn_merge(o_parts, lse_parts, out=out)
    torch.cuda.synchronize()
    ref_o, ref_lse = oracle.merge(o_parts.double().cpu().numpy(), lse_parts.double().cpu().numpy())
    got = o.float().cpu().numpy()
    bits = 8 if dtype == torch.bfloat16 else 24
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref_o), 1e-30))) - bits)
    assert (np.abs(got - ref_o) <= 1e-5 + ulp).all()
    lse_np = lse.cpu().numpy()
    finite = np.isfinite(ref_lse)
    assert np.isneginf(lse_np[~finite]).all() and (got[~finite] == 0).all()
    assert np.abs(lse_np[finite] - ref_lse[finite]).max() <= 1e-5


@pytest.mark.parametrize("L,Hq,Hkv,extra", [
    (3, 8, 1, {}),                                   # G = 8: 4 heads x 8 rows per tile
    (33, 8, 2, dict(window=500, sinks=4)),           # G = 4, 40-row head blocks
    (1, 8, 2, dict(pairing="interleaved")),
    (8, 16, 1, {}),                                  # G = 16: 8 heads x 8 rows
    (2, 6, 1, dict(mode="ntk", scale=4.0)),          # G = 6: 3 heads per tile
    (5, 4, 2, dict(split_qk=True, D=64)),            # split parts, D = 64
])
def test_splitkv_head_packed_decode(L, Hq, Hkv, extra):
    """Few queries per head: the kv group's heads share the two query tiles
    (head-packed layout); every head's rows against the oracle."""
    Lk = 2000
    w = W0.with_(Hq=Hq, Hkv=Hkv, **extra, L=Lk)
    q_all, k, v = make_inputs(w, device="cuda")
    q = q_all[:, :, Lk - L:]
    rope = rope_of(w)
    o, lse = run_split(q, k, v, rope, 4, window=w.window, sinks=w.sinks, q_offset=Lk - L,
                       split_qk=w.split_qk)
    ref = oracle_rows(q, k, v, rope, Lk - L, True, w.window, w.sinks)
    compare(o.float().cpu().numpy(), lse.cpu().numpy(), ref[0], ref[1])


@pytest.mark.parametrize("L,Lk,splits,extra", [
    (1, 1800, 2, dict(Hq=8, Hkv=2)),                 # 15 key tiles: splits of 8 and 7
    (1, 777, 7, dict(Hq=8, Hkv=2)),                  # one key tile per split: tile 1 gets none
    (2, 1000, 3, dict(Hq=6, Hkv=2)),                 # G = 3 (odd): packed only this way
    (1, 1500, 5, dict(Hq=2, Hkv=2)),                 # G = 1
    (4, 3000, 6, dict(Hq=8, Hkv=2, window=700, sinks=4)),
    (1, 2000, 4, dict(Hq=8, Hkv=2, k_prerotated=True)),
    # split QK^T: odd counts, one tile per split, keys split into their parts by
    # the rotate pass
    (1, 1800, 2, dict(Hq=8, Hkv=2, split_qk=True)),
    (2, 777, 13, dict(Hq=6, Hkv=2, split_qk=True)),
    (3, 2000, 5, dict(Hq=8, Hkv=2, split_qk=True, rotate_k_once=True)),
])
def test_splitkv_interleaved_key_tiles(L, Lk, splits, extra):
    """bf16 head-packed split-KV: both query tiles hold all G heads and take
    alternate key tiles of the split (two partial results per split); every
    head's rows against the oracle, edge counts of key tiles included.  With
    keys rotated on chip and G L <= 32, four softmax warps that hold no query
    help rotate the key tiles (256 rotating threads)."""
    extra = dict(extra)
    prerot = extra.pop("k_prerotated", False)
    once = extra.pop("rotate_k_once", False)
    w = W0.with_(**extra, L=Lk)
    q_all, k, v = make_inputs(w, device="cuda")
    q = q_all[:, :, Lk - L:]
    rope = rope_of(w)
    kk = lcx.apply_rope(k, rope) if prerot else k
    o, lse = run_split(q, kk, v, rope, splits, window=w.window, sinks=w.sinks, q_offset=Lk - L,
                       k_prerotated=prerot, split_qk=w.split_qk, rotate_k_once=once)
    ref = oracle_rows(q, k, v, rope, Lk - L, True, w.window, w.sinks)
    compare(o.float().cpu().numpy(), lse.cpu().numpy(), ref[0], ref[1])


@pytest.mark.parametrize("L,Lk,splits,extra", [
    (1, 2000, 5, dict(Hq=16, Hkv=4)),                          # G L = 4: 4 query columns
    (1, 2000, 5, dict(Hq=10, Hkv=2)),                          # G L = 5: 8 columns, 3 unused
    (2, 1500, 3, dict(Hq=8, Hkv=2, pairing="interleaved")),    # G L = 8
    (3, 3000, 6, dict(Hq=6, Hkv=2, window=900, sinks=5)),      # G L = 9: 16 columns
    (16, 2100, 4, dict(Hq=2, Hkv=2)),                          # G = 1, a 16-row chunk
    (1, 900, 12, dict(Hq=8, Hkv=2)),                           # 8 key tiles, 12 splits
    (1, 2000, 5, dict(Hq=8, Hkv=2, rotate_k_once=True)),       # keys rotated by the pass
    (1, 2000, 5, dict(Hq=8, Hkv=2, prerotated=True)),          # q and k arrive rotated
    (4, 1000, 3, dict(Hq=8, Hkv=2, causal=False)),
    # split QK^T (keys' fp16 and 8-bit parts and V in fp16 from the rotate pass)
    (1, 2000, 5, dict(Hq=8, Hkv=2, split_qk=True, rotate_k_once=True)),
    (2, 1500, 3, dict(Hq=8, Hkv=2, pairing="interleaved", split_qk=True, rotate_k_once=True)),
    (3, 3000, 6, dict(Hq=6, Hkv=2, window=900, sinks=5, split_qk=True, rotate_k_once=True)),
])
def test_splitkv_transposed_decode(L, Lk, splits, extra):
    """Key-split launches whose kv group holds at most 16 queries (bf16, D = 128,
    full rotary) run the transposed-score decode kernel: one key per TMEM lane
    and one query per column, 4, 8 or 16 columns read.  Every row of every head
    against the oracle, empty splits, both pairings and the rotated-input modes
    included."""
    extra = dict(extra)
    once = extra.pop("rotate_k_once", False)
    prerot = extra.pop("prerotated", False)
    causal = extra.pop("causal", True)
    w = W0.with_(**extra, L=Lk)
    q_all, k, v = make_inputs(w, device="cuda")
    rope = rope_of(w)
    q = q_all[:, :, Lk - L:]
    q_in, k_in = q, k
    if prerot:
        q_in = lcx.apply_rope(q_all, rope)[:, :, Lk - L:]
        k_in = lcx.apply_rope(k, rope)
    o, lse = run_split(q_in, k_in, v, rope, splits, causal=causal, window=w.window,
                       sinks=w.sinks, q_offset=Lk - L, prerotated=prerot, rotate_k_once=once,
                       split_qk=w.split_qk)
    ref = oracle_rows(q, k, v, rope, Lk - L, causal, w.window, w.sinks)
    compare(o.float().cpu().numpy(), lse.cpu().numpy(), ref[0], ref[1])


@pytest.mark.parametrize("splits", [4, 9])
def test_splitkv_decode_outlier_workload(splits):
    """A decode step of the outlier workload (8x outliers on 1% of the channels,
    YaRN s=8, a 4096-key window and 4 sinks) in its split-QK^T mode with the
    keys split once by the rotate pass: the transposed decode kernel's fp16 and
    e5m2 products against the oracle, every head, two batches."""
    w = WORKLOADS["sink_window_L65536"].with_(B=2, L=9000)
    q_all, k, v = make_inputs(w, device="cuda")
    q = q_all[:, :, w.L - 1:]
    rope = rope_of(w)
    o, lse = run_split(q, k, v, rope, splits, window=w.window, sinks=w.sinks,
                       q_offset=w.L - 1, split_qk=True, rotate_k_once=True)
    ref = oracle_rows(q, k, v, rope, w.L - 1, True, w.window, w.sinks)
    compare(o.float().cpu().numpy(), lse.cpu().numpy(), ref[0], ref[1])
