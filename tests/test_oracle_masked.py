"""Pins of the oracle's key-padding mask and dropout (oracle.masked), CPU only.

The generator is pinned to Philox4x32-10's published known answers; the draw
layout to its written definition; dropout to its statistics and to the closed
form of a single visible key; the key mask to the C oracle on the gathered keys
and to a loop written out on tiny inputs; p = 0 to the C oracle; the backward to
central differences of sum(O * dO) and to the identity sum_j P_ij dP_ij = dO_i . O_i.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from oracle import masked


def _rng_inputs(seed, B, Nq, Nk, H, d):
    rng = np.random.default_rng(seed)
    return (rng.normal(size=(B, Nq, H, d)), rng.normal(size=(B, Nk, H, d)), rng.normal(size=(B, Nk, H, d)),
            rng.normal(size=(B, Nq, H, d)))


def test_philox_known_answers(golden_dir):
    with open(os.path.join(golden_dir, "philox4x32_10_kat.json")) as f:
        kat = json.load(f)
    for vec in kat["vectors"]:
        c = [int(x, 16) for x in vec["counter"]]
        k = [int(x, 16) for x in vec["key"]]
        out = masked.philox4x32_10(*c, *k)
        assert ["%08x" % int(w) for w in out] == vec["out"]


def test_philox_vectorised_matches_scalar_calls():
    c0 = np.arange(5)
    out = masked.philox4x32_10(c0, 7, 11, 13, 0x1234, 0x5678)
    for n in range(5):
        one = masked.philox4x32_10(n, 7, 11, 13, 0x1234, 0x5678)
        assert [int(w[n]) for w in out] == [int(w) for w in one]


def test_draw_layout_as_documented():
    seed = (0x0123456789ABCDEF)
    b, h, i, j = 3, 5, 10, 7  # block (j // 2, i // 4) = (3, 2); word i % 4 = 2; odd key: high half
    words = masked.philox4x32_10(3, 2, 5, 3, 0x89ABCDEF, 0x01234567)
    assert int(masked.dropout_draws(seed, b, h, i, j)) == int(words[2]) >> 16
    assert int(masked.dropout_draws(seed, b, h, i, j - 1)) == int(words[2]) & 0xFFFF
    assert int(masked.dropout_draws(seed, b, h, i - 1, j)) == int(words[1]) >> 16


def test_threshold_rounding():
    assert masked.dropout_threshold(0.0) == 0
    assert masked.dropout_threshold(0.1) == 6554
    assert masked.dropout_threshold(0.5) == 32768
    with pytest.raises(ValueError):
        masked.dropout_threshold(1.0)


@pytest.mark.parametrize("p", [0.1, 0.5, 0.9])
def test_keep_rate_and_unbiased_scale(p):
    n = 1 << 20
    idx = np.arange(n)
    z = masked.dropout_scale(p, idx % 3, (idx // 3) % 5, (idx // 15) % 97, idx // 1455, seed=42)
    t = masked.dropout_threshold(p)
    keep_eff = 1.0 - t / 65536.0
    frac = float(np.mean(z > 0))
    sigma = math.sqrt(keep_eff * (1 - keep_eff) / n)
    assert abs(frac - keep_eff) < 6 * sigma
    assert abs(float(np.mean(z)) - 1.0) < 6 * sigma / keep_eff
    assert np.all((z == 0) | np.isclose(z, 1.0 / keep_eff, rtol=0, atol=1e-15))


def test_draws_are_uniform_over_16_bits():
    n = 1 << 20
    idx = np.arange(n)
    u = masked.dropout_draws(7, 0, idx % 11, idx // 11 % 1000, idx // 11000)
    counts = np.bincount(u >> 12, minlength=16)  # 16 bins
    expected = n / 16
    chi2 = float(((counts - expected) ** 2 / expected).sum())
    assert chi2 < 50  # 15 degrees of freedom: P(chi2 > 50) ~ 1e-5


@pytest.mark.parametrize("causal", [False, True])
def test_p_zero_no_mask_is_the_plain_oracle(causal):
    q, k, v, _ = _rng_inputs(1, 2, 37, 53, 2, 8)
    o, lse = masked.attn_fwd_masked(q, k, v, causal, 0.3)
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, causal, 0.3)
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, rtol=1e-13, atol=1e-12)


def test_key_mask_equals_gathering_the_kept_keys():
    q, k, v, _ = _rng_inputs(2, 2, 20, 30, 3, 8)
    rng = np.random.default_rng(3)
    mask = rng.random((2, 30)) < 0.6
    o, lse = masked.attn_fwd_masked(q, k, v, False, 0.4, key_mask=mask)
    for b in range(2):
        keep = np.flatnonzero(mask[b])
        ob, lb = oracle.attn_fwd(q[b:b + 1], k[b:b + 1, keep], v[b:b + 1, keep], False, 0.4)
        np.testing.assert_allclose(o[b], ob[0], rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[b], lb[0], rtol=1e-13, atol=1e-12)


def test_causal_mask_and_dropout_by_hand():
    q, k, v, _ = _rng_inputs(4, 1, 5, 7, 1, 3)
    mask = np.array([[True, False, True, True, False, True, True]])
    p, seed, scale = 0.3, 99, 0.7
    o, lse = masked.attn_fwd_masked(q, k, v, True, scale, key_mask=mask, dropout_p=p, seed=seed)
    t = masked.dropout_threshold(p)
    for i in range(5):
        num, den, mx = np.zeros(3), 0.0, -math.inf
        keys = [j for j in range(7) if mask[0, j] and j <= i + 2]
        for j in keys:
            mx = max(mx, scale * float(q[0, i, 0] @ k[0, j, 0]))
        for j in keys:
            w = math.exp(scale * float(q[0, i, 0] @ k[0, j, 0]) - mx)
            den += w
            word = masked.philox4x32_10(j // 2, i // 4, 0, 0, seed, 0)[i % 4]
            draw = (int(word) >> 16) if j % 2 else (int(word) & 0xFFFF)
            num += (w * (65536.0 / (65536.0 - t)) if draw >= t else 0.0) * v[0, j, 0]
        np.testing.assert_allclose(o[0, i, 0], num / den, rtol=1e-12, atol=1e-13)
        assert abs(lse[0, 0, i] - (mx + math.log(den))) < 1e-12


def test_fully_masked_rows():
    q, k, v, _ = _rng_inputs(5, 1, 4, 4, 2, 8)
    mask = np.array([[False, False, True, True]])
    o, lse = masked.attn_fwd_masked(q, k, v, True, 0.5, key_mask=mask, dropout_p=0.2, seed=1)
    assert np.all(o[0, :2] == 0) and np.all(np.isneginf(lse[0, :, :2]))
    assert np.all(np.isfinite(lse[0, :, 2:]))


def test_single_visible_key_closed_form():
    q, k, v, _ = _rng_inputs(6, 1, 64, 1, 2, 4)
    p, seed = 0.25, 5
    o, _ = masked.attn_fwd_masked(q, k, v, False, 0.5, dropout_p=p, seed=seed)
    for h in range(2):
        z = masked.dropout_scale(p, 0, h, np.arange(64), 0, seed)
        np.testing.assert_allclose(o[0, :, h], z[:, None] * v[0, 0, h][None, :], rtol=0, atol=1e-15)
    assert 0 < np.count_nonzero(o[0, :, 0, 0] == 0) < 64  # some rows dropped, some kept


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("p", [0.0, 0.4])
def test_backward_finite_differences(causal, p):
    q, k, v, dout = _rng_inputs(7, 1, 6, 5, 2, 3)
    mask = np.array([[True, True, False, True, True]])
    args = dict(key_mask=mask, dropout_p=p, seed=11)
    grads = masked.attn_bwd_masked(q, k, v, dout, causal, 0.8, **args)
    h = 1e-6
    for x, g in zip((q, k, v), grads):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            x0 = x[idx]
            x[idx] = x0 + h
            lp = float(np.sum(masked.attn_fwd_masked(q, k, v, causal, 0.8, **args)[0] * dout))
            x[idx] = x0 - h
            lm = float(np.sum(masked.attn_fwd_masked(q, k, v, causal, 0.8, **args)[0] * dout))
            x[idx] = x0
            num[idx] = (lp - lm) / (2 * h)
        assert np.max(np.abs(num - g)) <= 1e-6 * max(1.0, np.max(np.abs(g)))


def test_backward_p_zero_is_the_plain_oracle():
    q, k, v, dout = _rng_inputs(8, 2, 19, 23, 2, 8)
    g = masked.attn_bwd_masked(q, k, v, dout, True, 0.35)
    r = oracle.attn_bwd(q, k, v, dout, True, 0.35)
    for a, b in zip(g, r):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def test_row_term_identity_with_dropout():
    # sum_j P_ij dP_ij = dO_i . O_i holds with the dropped, rescaled P as well
    q, k, v, dout = _rng_inputs(9, 1, 16, 16, 1, 8)
    p, seed, scale = 0.3, 3, 0.5
    o, _ = masked.attn_fwd_masked(q, k, v, True, scale, dropout_p=p, seed=seed)
    vis = np.tril(np.ones((16, 16), dtype=bool))
    s = np.where(vis, scale * q[0, :, 0] @ k[0, :, 0].T, -np.inf)
    pr = np.exp(s - s.max(axis=1, keepdims=True))
    pr /= pr.sum(axis=1, keepdims=True)
    ii, jj = np.meshgrid(np.arange(16), np.arange(16), indexing="ij")
    z = masked.dropout_scale(p, 0, 0, ii, jj, seed)
    dp = z * (dout[0, :, 0] @ v[0, :, 0].T)
    np.testing.assert_allclose((pr * dp).sum(axis=1), (dout[0, :, 0] * o[0, :, 0]).sum(axis=1), rtol=1e-12,
                               atol=1e-12)


# ---------------------------------------------------------------- block-sparse


@pytest.mark.parametrize("causal", [False, True])
def test_all_ones_block_mask_changes_nothing(causal):
    q, k, v, _ = _rng_inputs(10, 2, 20, 20, 2, 8)
    bm = np.ones((3, 3), dtype=bool)
    o, lse = masked.attn_fwd_masked(q, k, v, causal, 0.3, block_mask=bm, block=(8, 8))
    o2, lse2 = masked.attn_fwd_masked(q, k, v, causal, 0.3)
    assert np.array_equal(o, o2) and np.array_equal(lse, lse2)


def test_block_diagonal_mask_is_attention_within_each_block():
    q, k, v, _ = _rng_inputs(11, 1, 24, 24, 2, 8)
    bm = np.eye(3, dtype=bool)  # blocks of 8: three independent 8-token problems
    o, lse = masked.attn_fwd_masked(q, k, v, False, 0.5, block_mask=bm, block=(8, 8))
    for blk in range(3):
        sl = slice(8 * blk, 8 * blk + 8)
        ob, lb = oracle.attn_fwd(q[:, sl], k[:, sl], v[:, sl], False, 0.5)
        np.testing.assert_allclose(o[:, sl], ob, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[:, :, sl], lb, rtol=1e-13, atol=1e-12)


def test_column_pattern_equals_the_key_mask():
    q, k, v, _ = _rng_inputs(12, 1, 12, 16, 3, 4)
    cols = np.array([True, False, True, True])  # key blocks of 4
    bm = np.tile(cols, (3, 1))  # 3 query blocks of 4
    o, lse = masked.attn_fwd_masked(q, k, v, True, 0.6, block_mask=bm, block=(4, 4))
    o2, lse2 = masked.attn_fwd_masked(q, k, v, True, 0.6, key_mask=np.repeat(cols, 4)[None, :])
    assert np.array_equal(o, o2) and np.array_equal(lse, lse2)


def test_per_head_block_masks():
    q, k, v, _ = _rng_inputs(13, 1, 8, 8, 2, 4)
    bm = np.array([[[1, 0], [1, 1]], [[1, 1], [0, 1]]], dtype=bool)  # [H, 2, 2], blocks of 4
    o, _ = masked.attn_fwd_masked(q, k, v, False, 0.5, block_mask=bm, block=(4, 4))
    for h in range(2):
        oh, _ = masked.attn_fwd_masked(q[:, :, h:h + 1], k[:, :, h:h + 1], v[:, :, h:h + 1], False, 0.5,
                                       block_mask=bm[h], block=(4, 4))
        assert np.array_equal(o[:, :, h], oh[:, :, 0])
    # head 0, query block 0 sees only key block 0: a 4-key problem
    ob, _ = oracle.attn_fwd(q[:, :4, :1], k[:, :4, :1], v[:, :4, :1], False, 0.5)
    np.testing.assert_allclose(o[:, :4, :1], ob, rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_block_sparse_backward_finite_differences(causal):
    q, k, v, dout = _rng_inputs(14, 1, 6, 6, 1, 3)
    bm = np.array([[1, 0, 1], [1, 1, 0], [0, 1, 1]], dtype=bool)  # blocks of 2
    args = dict(block_mask=bm, block=(2, 2), dropout_p=0.25, seed=4)
    grads = masked.attn_bwd_masked(q, k, v, dout, causal, 0.9, **args)
    h = 1e-6
    for x, g in zip((q, k, v), grads):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            x0 = x[idx]
            x[idx] = x0 + h
            lp = float(np.sum(masked.attn_fwd_masked(q, k, v, causal, 0.9, **args)[0] * dout))
            x[idx] = x0 - h
            lm = float(np.sum(masked.attn_fwd_masked(q, k, v, causal, 0.9, **args)[0] * dout))
            x[idx] = x0
            num[idx] = (lp - lm) / (2 * h)
        assert np.max(np.abs(num - g)) <= 1e-6 * max(1.0, np.max(np.abs(g)))
