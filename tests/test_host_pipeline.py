"""Host logic of attn_fwd_host's pipeline (no GPU): the pieces it cuts a call
into cover every (batch, kv head, query row) exactly once, query cuts sit on
128-row blocks (so every query tile starts where it does in one call over
everything), and causal prefill's first and last pieces are the short ones."""
import itertools

import numpy as np
import pytest

import ntk_rope_flashattn_b200 as lcx


def coverage(pieces, B, Hkv, L):
    seen = np.zeros((B, Hkv, L), dtype=np.int32)
    for b, g0, g1, i0, i1 in pieces:
        bs = range(B) if b is None else [b]
        for bb in bs:
            seen[bb, g0:g1, i0:i1] += 1
    return seen


@pytest.mark.parametrize("B,Hkv,L,chunks,causal", [
    (b, h, L, c, causal)
    for b, h, L, c, causal in itertools.product((1, 2, 3), (1, 2, 8), (1, 129, 511, 512, 600,
                                                                      1100, 131072),
                                                (1, 3, 8), (True, False))
])
def test_pieces_cover_every_row_once(B, Hkv, L, chunks, causal):
    pieces = lcx.host_pieces(B, Hkv, L, chunks, causal=causal)
    assert (coverage(pieces, B, Hkv, L) == 1).all()
    for b, g0, g1, i0, i1 in pieces:
        assert 0 <= g0 < g1 <= Hkv and 0 <= i0 < i1 <= L
        assert i0 % 128 == 0 and (i1 == L or i1 % 128 == 0)
        if not causal:
            assert (i0, i1) == (0, L)


def test_causal_first_and_last_pieces_are_short():
    L = 131072
    pieces = lcx.host_pieces(1, 8, L, 8)
    assert pieces[0][3:] == (0, L // 4) and pieces[1][3:] == (L // 4, L)
    assert pieces[-1][3:] == (3 * L // 4, L) and pieces[-2][3:] == (0, 3 * L // 4)
    assert pieces[0][:3] == pieces[1][:3] and pieces[-1][:3] == pieces[-2][:3]
    assert len(pieces) == 8 + 2
    # a single group: first quarter, middle, last quarter
    one = lcx.host_pieces(1, 1, 1100, 1)
    assert [p[3:] for p in one] == [(0, 256), (256, 768), (768, 1100)]


def test_no_query_cuts_when_they_do_not_apply():
    assert all(p[3:] == (0, 300) for p in lcx.host_pieces(2, 4, 300, 8))      # under 512 rows
    assert all(p[3:] == (0, 4096) for p in lcx.host_pieces(1, 8, 4096, 8, q_offset=100))
    assert lcx.host_pieces(2, 8, 4096, 8, one_piece=True) == [(None, 0, 8, 0, 4096)]
