"""Host logic of the binding (CPU).

- The host-buffer calls (forward_from_host, backward_from_host) cut a problem into independent
  pieces whose copies overlap the neighbouring pieces' kernels.  Every piece must be a
  contiguous block of every tensor; the pieces must cover the problem exactly once; and for
  B == 1 a piece must hold whole GQA groups (its query heads are exactly those of its KV heads),
  so that each piece is an attention problem of its own.
"""
import numpy as np
import pytest

import tiled_attention_forward_03_b200 as attn


def _covered(sl, n):
    start = 0 if sl.start is None else sl.start
    stop = n if sl.stop is None else sl.stop
    return list(range(start, stop))


@pytest.mark.parametrize("B,Hq,Hkv,n", [
    (4, 16, 16, 4), (4, 16, 16, 8), (3, 8, 2, 4), (16, 16, 16, 4), (2, 32, 8, 1), (5, 4, 1, 3),
    (1, 32, 8, 4), (1, 32, 8, 3), (1, 8, 8, 16), (1, 4, 1, 4), (1, 2, 2, 1), (7, 6, 3, 100),
])
def test_pieces_partition_the_problem(B, Hq, Hkv, n):
    pieces = attn._pieces(B, Hq, Hkv, n)
    assert 1 <= len(pieces) <= n
    g = Hq // Hkv
    seen_q, seen_kv = [], []
    for b_sl, q_sl, kv_sl in pieces:
        bs = _covered(b_sl, B)
        qs = _covered(q_sl, Hq)
        ks = _covered(kv_sl, Hkv)
        assert bs and qs and ks
        # contiguous ranges (a slice with step 1)
        assert b_sl.step in (None, 1) and q_sl.step in (None, 1) and kv_sl.step in (None, 1)
        # whole GQA groups: the query heads are exactly those of the KV heads
        assert qs == [h for kh in ks for h in range(kh * g, (kh + 1) * g)]
        seen_q += [(b, h) for b in bs for h in qs]
        seen_kv += [(b, h) for b in bs for h in ks]
    assert sorted(seen_q) == [(b, h) for b in range(B) for h in range(Hq)]
    assert sorted(seen_kv) == [(b, h) for b in range(B) for h in range(Hkv)]
    assert len(set(seen_q)) == len(seen_q)


def test_pieces_use_batch_rows_when_there_are_several():
    pieces = attn._pieces(8, 16, 4, 4)
    assert len(pieces) == 4
    assert all(q == slice(None) and kv == slice(None) for _, q, kv in pieces)
    assert [(_covered(b, 8)) for b, _, _ in pieces] == [[0, 1], [2, 3], [4, 5], [6, 7]]


def test_single_batch_row_is_cut_by_kv_head_groups():
    pieces = attn._pieces(1, 32, 8, 4)
    assert [(_covered(kv, 8), _covered(q, 32)) for _, q, kv in pieces] == [
        ([0, 1], list(range(0, 8))), ([2, 3], list(range(8, 16))),
        ([4, 5], list(range(16, 24))), ([6, 7], list(range(24, 32)))]
