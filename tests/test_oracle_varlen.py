"""Pins of the oracle's variable-length forward (oracle.attn_fwd_varlen), CPU only.

Packing sequences without padding changes where rows live, not what attention
computes: a one-sequence batch is the dense forward; equal-length sequences are
the dense batch; reordering the sequences only moves their output blocks; and a
direct softmax of one row written out here in numpy agrees in fp64.
"""
import numpy as np
import pytest

import oracle
from exact_io_aware_54_b200 import synth


def _f64(t):
    return t.double().numpy()


def _pack(seed, lq, lk, H, d):
    q = _f64(synth._normal((sum(lq), H, d), seed))
    k = _f64(synth._normal((sum(lk), H, d), seed + 1))
    v = _f64(synth._normal((sum(lk), H, d), seed + 2))
    cq = np.concatenate([[0], np.cumsum(lq)]).astype(np.int32)
    ck = np.concatenate([[0], np.cumsum(lk)]).astype(np.int32)
    return q, k, v, cq, ck


@pytest.mark.parametrize("causal", [False, True])
def test_single_sequence_is_dense_forward(causal):
    q, k, v, cq, ck = _pack(81, [37], [53], 2, 64)
    o, lse = oracle.attn_fwd_varlen(q, k, v, cq, ck, causal, 0.125)
    od, ld = oracle.attn_fwd(q[None], k[None], v[None], causal, 0.125)
    assert np.array_equal(o, od[0]) and np.array_equal(lse, ld[0])


@pytest.mark.parametrize("causal", [False, True])
def test_equal_lengths_are_the_dense_batch(causal):
    q, k, v, cq, ck = _pack(82, [40, 40, 40], [70, 70, 70], 2, 64)
    o, lse = oracle.attn_fwd_varlen(q, k, v, cq, ck, causal, 0.2)
    od, ld = oracle.attn_fwd(q.reshape(3, 40, 2, 64), k.reshape(3, 70, 2, 64), v.reshape(3, 70, 2, 64), causal, 0.2)
    assert np.array_equal(o, od.reshape(120, 2, 64))
    assert np.array_equal(lse, np.concatenate(list(ld), axis=1))


def test_reordering_sequences_moves_blocks():
    lq, lk = [5, 30, 1, 17], [9, 30, 4, 40]
    q, k, v, cq, ck = _pack(83, lq, lk, 3, 64)
    o, lse = oracle.attn_fwd_varlen(q, k, v, cq, ck, True, 0.125)
    order = [2, 0, 3, 1]
    q2 = np.concatenate([q[cq[b]:cq[b + 1]] for b in order])
    k2 = np.concatenate([k[ck[b]:ck[b + 1]] for b in order])
    v2 = np.concatenate([v[ck[b]:ck[b + 1]] for b in order])
    cq2 = np.concatenate([[0], np.cumsum([lq[b] for b in order])]).astype(np.int32)
    ck2 = np.concatenate([[0], np.cumsum([lk[b] for b in order])]).astype(np.int32)
    o2, lse2 = oracle.attn_fwd_varlen(q2, k2, v2, cq2, ck2, True, 0.125)
    for i, b in enumerate(order):
        assert np.array_equal(o2[cq2[i]:cq2[i + 1]], o[cq[b]:cq[b + 1]])
        assert np.array_equal(lse2[:, cq2[i]:cq2[i + 1]], lse[:, cq[b]:cq[b + 1]])


def test_one_row_by_hand_bottom_right_causal():
    lq, lk = [3, 6], [2, 10]
    q, k, v, cq, ck = _pack(84, lq, lk, 1, 64)
    o, lse = oracle.attn_fwd_varlen(q, k, v, cq, ck, True, 0.3)
    # sequence 1, its row 1: bottom-right alignment sees keys 0 .. 1 + (10 - 6) = 5
    row = cq[1] + 1
    keys = k[ck[1]:ck[1] + 6, 0]
    vals = v[ck[1]:ck[1] + 6, 0]
    s = 0.3 * keys @ q[row, 0]
    w = np.exp(s - s.max())
    np.testing.assert_allclose(o[row, 0], (w[:, None] * vals).sum(0) / w.sum(), rtol=1e-12, atol=1e-12)
    assert abs(lse[0, row] - (s.max() + np.log(w.sum()))) < 1e-12


def test_empty_sequences():
    q, k, v, cq, ck = _pack(85, [0, 4, 3], [5, 0, 2], 2, 64)
    o, lse = oracle.attn_fwd_varlen(q, k, v, cq, ck, False, 0.125)
    assert np.all(o[0:4] == 0) and np.all(np.isneginf(lse[:, 0:4]))  # sequence 1 has no keys
    assert np.all(np.isfinite(lse[:, 4:7]))


# ---------------------------------------------------------------- backward
# The gradients of the packed loss sum(O * dO) are pinned by central differences of
# the packed forward (a gradient that leaked across sequences, dropped a term or
# mis-aligned the causal mask would miss them), by the softmax identity
# sum_j dS_ij = 0 (so the keys' dK of one sequence and head sum to zero), and by the
# rows that take no part in the loss.


def _packed_loss(q, k, v, dout, cq, ck, causal, scale):
    o, _ = oracle.attn_fwd_varlen(q, k, v, cq, ck, causal, scale)
    return float(np.sum(o * dout))


@pytest.mark.parametrize("causal", [False, True])
def test_backward_finite_differences(causal):
    rng = np.random.default_rng(86)
    lq, lk, H, d, scale, h = [2, 0, 3, 4], [3, 2, 1, 2], 2, 3, 0.7, 1e-6
    q = rng.normal(size=(sum(lq), H, d))
    k = rng.normal(size=(sum(lk), H, d))
    v = rng.normal(size=(sum(lk), H, d))
    dout = rng.normal(size=(sum(lq), H, d))
    cq = np.concatenate([[0], np.cumsum(lq)]).astype(np.int32)
    ck = np.concatenate([[0], np.cumsum(lk)]).astype(np.int32)
    grads = oracle.attn_bwd_varlen(q, k, v, dout, cq, ck, causal, scale)
    for x, g in zip((q, k, v), grads):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            x0 = x[idx]
            x[idx] = x0 + h
            lp = _packed_loss(q, k, v, dout, cq, ck, causal, scale)
            x[idx] = x0 - h
            lm = _packed_loss(q, k, v, dout, cq, ck, causal, scale)
            x[idx] = x0
            num[idx] = (lp - lm) / (2 * h)
        assert np.max(np.abs(num - g)) <= 1e-6 * max(1.0, np.max(np.abs(g)))


@pytest.mark.parametrize("causal", [False, True])
def test_backward_dk_sums_to_zero_per_sequence(causal):
    lq, lk = [7, 20, 1], [9, 20, 5]
    q, k, v, cq, ck = _pack(87, lq, lk, 2, 16)
    dout = _f64(synth._normal(q.shape, 90))
    _, dk, _ = oracle.attn_bwd_varlen(q, k, v, dout, cq, ck, causal, 0.25)
    for b in range(3):
        s = dk[ck[b]:ck[b + 1]].sum(axis=0)
        assert np.max(np.abs(s)) <= 1e-12 * max(1.0, np.max(np.abs(dk)))


def test_backward_rows_outside_the_loss_are_zero():
    # sequence 0 has keys but no queries, sequence 1 queries but no keys, and the
    # packed buffers end with rows that belong to no sequence
    lq, lk = [0, 3, 4], [5, 0, 6]
    q, k, v, cq, ck = _pack(88, lq + [2], lk + [3], 2, 8)
    cq, ck = cq[:-1], ck[:-1]
    dout = _f64(synth._normal(q.shape, 91))
    dq, dk, dv = oracle.attn_bwd_varlen(q, k, v, dout, cq, ck, True, 0.3)
    assert np.all(dk[0:5] == 0) and np.all(dv[0:5] == 0)
    assert np.all(dq[0:3] == 0)
    assert np.all(dq[7:] == 0) and np.all(dk[11:] == 0) and np.all(dv[11:] == 0)
    assert np.any(dq[3:7] != 0) and np.any(dk[5:11] != 0) and np.any(dv[5:11] != 0)
