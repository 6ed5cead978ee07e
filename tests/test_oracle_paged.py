"""Pins of the oracle's paged decode (oracle.decode_paged), CPU only.

A paged cache changes where each key lives, not what decode computes ("Flash
Attention saves IO, not N^2 work", section 6 names paging as the batched-decode
layout question).  The pins: an in-order page table reproduces the packed decode
bit for bit; moving pages around in the cache (and the table with them) changes
nothing; and a direct per-key evaluation that follows the page lookups by hand,
independent of the oracle's C code, agrees in fp64.
"""
import numpy as np
import pytest

import oracle
from exact_io_aware_54_b200 import synth


def _f64(t):
    return t.double().numpy()


def _paginate(k, v, cu, page_size):
    """Packed [total, H, d] -> in-order pages and table (test helper)."""
    lens = np.diff(cu)
    B = len(lens)
    H, d = k.shape[1], k.shape[2]
    ppseq = [(int(L) + page_size - 1) // page_size for L in lens]
    table = np.full((B, max(1, max(ppseq))), -1, dtype=np.int32)
    kp = np.zeros((sum(ppseq), page_size, H, d))
    vp = np.zeros_like(kp)
    nxt = 0
    for b, L in enumerate(lens):
        for pg in range(ppseq[b]):
            lo = cu[b] + pg * page_size
            hi = min(cu[b] + L, lo + page_size)
            kp[nxt, :hi - lo] = k[lo:hi]
            vp[nxt, :hi - lo] = v[lo:hi]
            table[b, pg] = nxt
            nxt += 1
    return kp, vp, table, lens.astype(np.int32)


@pytest.mark.parametrize("page_size", [1, 7, 16, 64])
def test_in_order_pages_equal_packed_decode(page_size):
    lengths = [0, 1, 15, 16, 17, 130]
    q, k, v, cu = synth.decode_inputs(61, lengths, 3, 64)
    q, k, v, cu = _f64(q), _f64(k), _f64(v), cu.numpy()
    o_ref, lse_ref = oracle.decode(q, k, v, cu, 0.125)
    kp, vp, table, lens = _paginate(k, v, cu, page_size)
    o, lse = oracle.decode_paged(q, kp, vp, table, lens, 0.125)
    assert np.array_equal(o, o_ref)
    assert np.array_equal(lse, lse_ref)


def test_moving_pages_changes_nothing():
    q, kp, vp, table, lens = synth.paged_decode_inputs(62, [5, 40, 33, 0, 64], 2, 64, 16)
    q, kp, vp, table, lens = _f64(q), _f64(kp), _f64(vp), table.numpy(), lens.numpy()
    o1, l1 = oracle.decode_paged(q, kp, vp, table, lens, 0.125)
    perm = np.random.default_rng(7).permutation(kp.shape[0])  # new slot of each page
    kp2, vp2 = np.empty_like(kp), np.empty_like(vp)
    kp2[perm], vp2[perm] = kp, vp
    table2 = np.where(table >= 0, perm[np.maximum(table, 0)], -1).astype(np.int32)
    o2, l2 = oracle.decode_paged(q, kp2, vp2, table2, lens, 0.125)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_matches_hand_walk_of_the_page_table():
    """Softmax over the keys found by walking the table key by key, in numpy."""
    page_size = 8
    q, kp, vp, table, lens = synth.paged_decode_inputs(63, [1, 9, 23], 2, 64, page_size)
    q, kp, vp, table, lens = _f64(q), _f64(kp), _f64(vp), table.numpy(), lens.numpy()
    scale = 0.3
    o, lse = oracle.decode_paged(q, kp, vp, table, lens, scale)
    for b in range(len(lens)):
        for h in range(q.shape[1]):
            keys, vals = [], []
            for t in range(int(lens[b])):
                page, row = table[b][t // page_size], t % page_size
                keys.append(kp[page, row, h])
                vals.append(vp[page, row, h])
            s = scale * np.array(keys) @ q[b, h]
            m = s.max()
            w = np.exp(s - m)
            np.testing.assert_allclose(o[b, h], (w[:, None] * np.array(vals)).sum(0) / w.sum(), rtol=1e-12,
                                       atol=1e-12)
            assert abs(lse[b, h] - (m + np.log(w.sum()))) < 1e-12


def test_empty_sequences():
    q, kp, vp, table, lens = synth.paged_decode_inputs(64, [0, 0], 2, 64, 16)
    o, lse = oracle.decode_paged(_f64(q), _f64(kp), _f64(vp), table.numpy(), lens.numpy(), 0.125)
    assert np.all(o == 0) and np.all(np.isneginf(lse))
