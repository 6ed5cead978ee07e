"""Key-padding mask and dropout for the fp64 oracle -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may use this module; it shares no code with the CUDA path.

What it computes.  The pages name a padding mask and dropout among the semantics
a fused attention kernel has to match, with dropout's random mask generated again
in the backward pass instead of being stored ("FlashAttention saves IO, not N^2
work", section 8, the verification checklist; "AI Bible 13", section 03, masks and
dropout fused into the one kernel).  They give no formulas for either, so this
module takes the plain textbook reading:

* key-padding mask: key j of batch element b takes part iff key_mask[b, j]; it is
  excluded like a causally masked key (its score is -inf), on top of the causal
  mask when both are set.  A row with no key left has O = 0 and lse = -inf.
* block-sparse attention (the block-sparse variant the second page credits with
  reaching 64K tokens, "AI Bible 13", section 05): a 0/1 matrix over (query
  block, key block) of block_q x block_k elements; a zero block excludes all its
  keys from its queries, on top of the other masks.
* dropout with probability p acts on the normalised probabilities: with the
  statistics m, l and lse of the undropped row,
      O_i = sum_j P_ij z_ij v_j,   z_ij = keep_ij / (1 - p_eff),
  so lse is that of the undropped softmax (what the backward pass keeps).
* backward: the vector-Jacobian product of sum(O * dO) through the same z:
      dV_j = sum_i P_ij z_ij dO_i,   dP_ij = z_ij (dO_i . v_j),
      D_i = sum_j P_ij dP_ij,   dS_ij = P_ij (dP_ij - D_i),
      dQ_i = scale sum_j dS_ij k_j,   dK_j = scale sum_i dS_ij q_i.

The random mask (a reading of this build; the pages fix no generator).  keep_ij
comes from Philox4x32-10 (Salmon, Moraes, Dror and Shaw, "Parallel random
numbers: as easy as 1, 2, 3", SC'11), keyed by the 64-bit seed (low word first)
with counter (j // 2, i // 4, h, b).  One call yields four 32-bit words for a
block of 4 queries x 2 keys: query i uses word i % 4, key j its low (j even) or
high (j odd) 16 bits.  The element is kept iff those 16 bits are >= t, where
t = round(p * 65536); p_eff = t / 65536.  In a packed variable-length batch b is
the sequence and i, j count from the sequence's first row.
"""
from __future__ import annotations

import numpy as np

_MASK32 = np.uint64(0xFFFFFFFF)
_PHILOX_M0 = np.uint64(0xD2511F53)
_PHILOX_M1 = np.uint64(0xCD9E8D57)
_PHILOX_W0 = np.uint64(0x9E3779B9)
_PHILOX_W1 = np.uint64(0xBB67AE85)


def philox4x32_10(c0, c1, c2, c3, k0: int, k1: int):
    """Philox4x32 with 10 rounds (Salmon et al., SC'11).  Counters are arrays (or
    scalars) of 32-bit values, broadcast together; returns four uint32 arrays."""
    c = [np.asarray(x, dtype=np.uint64) & _MASK32 for x in (c0, c1, c2, c3)]
    c = list(np.broadcast_arrays(*c))
    key0, key1 = np.uint64(k0 & 0xFFFFFFFF), np.uint64(k1 & 0xFFFFFFFF)
    for r in range(10):
        if r:  # the key schedule: add the two Weyl constants
            key0 = (key0 + _PHILOX_W0) & _MASK32
            key1 = (key1 + _PHILOX_W1) & _MASK32
        p0 = _PHILOX_M0 * c[0]  # 32 x 32 -> 64-bit products (exact in uint64)
        p1 = _PHILOX_M1 * c[2]
        c = [(p1 >> np.uint64(32)) ^ c[1] ^ key0, p1 & _MASK32, (p0 >> np.uint64(32)) ^ c[3] ^ key1,
             p0 & _MASK32]
    return [x.astype(np.uint32) for x in c]


def dropout_threshold(p: float) -> int:
    """t = round(p * 65536): an element is dropped when its 16-bit draw is below t."""
    if not 0.0 <= p < 1.0:
        raise ValueError("dropout probability must be in [0, 1)")
    return int(np.floor(p * 65536.0 + 0.5))


def dropout_draws(seed: int, b, h, i, j):
    """The 16-bit draw of element (b, h, i, j) (arrays broadcast together)."""
    b, h, i, j = (np.asarray(x, dtype=np.int64) for x in (b, h, i, j))
    words = philox4x32_10(j >> 1, i >> 2, h, b, seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF)
    w = np.choose(i & 3, words)
    return np.where((j & 1) == 0, w & np.uint32(0xFFFF), w >> np.uint32(16)).astype(np.uint32)


def dropout_scale(p: float, b, h, i, j, seed: int):
    """z = keep / (1 - p_eff) for the elements (b, h, i, j), fp64."""
    t = dropout_threshold(p)
    if t == 0:
        return np.ones(np.broadcast(np.asarray(b), np.asarray(h), np.asarray(i), np.asarray(j)).shape)
    keep = dropout_draws(seed, b, h, i, j) >= t
    return keep * (65536.0 / (65536.0 - t))


def _visible(Nq, Nk, causal, key_mask_b, block_mask_bh=None, block=(128, 128)):
    """[Nq, Nk] boolean: key j takes part in row i."""
    vis = np.ones((Nq, Nk), dtype=bool)
    if causal:
        vis &= np.arange(Nk)[None, :] <= np.arange(Nq)[:, None] + (Nk - Nq)
    if key_mask_b is not None:
        vis &= np.asarray(key_mask_b, dtype=bool)[None, :]
    if block_mask_bh is not None:
        bm = np.asarray(block_mask_bh, dtype=bool)
        vis &= bm[np.arange(Nq)[:, None] // block[0], np.arange(Nk)[None, :] // block[1]]
    return vis


def _block_mask_of(block_mask, b, h):
    """The [n_qblocks, n_kblocks] mask of head (b, h) from a [nq, nk], [H, nq, nk]
    or [B, H, nq, nk] array (None: no block mask)."""
    if block_mask is None:
        return None
    bm = np.asarray(block_mask)
    if bm.ndim == 2:
        return bm
    if bm.ndim == 3:
        return bm[h]
    return bm[b, h]


def _head_probs(qh, kh, scale, vis):
    """Safe softmax of one head's scores (max, sum, normalise); P = 0 and lse = -inf
    on rows with no visible key."""
    s = scale * (qh @ kh.T)
    s = np.where(vis, s, -np.inf)
    m = s.max(axis=1, initial=-np.inf)
    empty = ~np.isfinite(m)
    m_safe = np.where(empty, 0.0, m)
    e = np.where(vis, np.exp(s - m_safe[:, None]), 0.0)
    l = e.sum(axis=1)
    p = np.where(empty[:, None], 0.0, e / np.where(empty, 1.0, l)[:, None])
    lse = np.where(empty, -np.inf, m_safe + np.log(np.where(empty, 1.0, l)))
    return p, lse


def attn_fwd_masked(q, k, v, causal: bool, scale: float, key_mask=None, dropout_p: float = 0.0, seed: int = 0,
                    block_mask=None, block=(128, 128)):
    """q [B, Nq, H, d], k, v [B, Nk, H, d]; key_mask [B, Nk] bool or None; block_mask
    over (query block, key block) of `block` = (block_q, block_k) elements, shared
    ([nq, nk]), per head ([H, nq, nk]) or per (b, h) ([B, H, nq, nk]), or None ->
    (o [B, Nq, H, d], lse [B, H, Nq]) in fp64."""
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    B, Nq, H, d = q.shape
    Nk = k.shape[1]
    o = np.zeros((B, Nq, H, v.shape[3]))
    lse = np.full((B, H, Nq), -np.inf)
    ii, jj = np.meshgrid(np.arange(Nq), np.arange(Nk), indexing="ij")
    for b in range(B):
        for h in range(H):
            vis = _visible(Nq, Nk, causal, None if key_mask is None else key_mask[b],
                           _block_mask_of(block_mask, b, h), block)
            p, lse[b, h] = _head_probs(q[b, :, h], k[b, :, h], scale, vis)
            z = dropout_scale(dropout_p, b, h, ii, jj, seed)
            o[b, :, h] = (p * z) @ v[b, :, h]
    return o, lse


def attn_bwd_masked(q, k, v, dout, causal: bool, scale: float, key_mask=None, dropout_p: float = 0.0,
                    seed: int = 0, block_mask=None, block=(128, 128)):
    """Gradients of sum(O * dout) for `attn_fwd_masked`; returns (dq, dk, dv) in fp64."""
    q, k, v, dout = (np.asarray(x, dtype=np.float64) for x in (q, k, v, dout))
    B, Nq, H, d = q.shape
    Nk = k.shape[1]
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    ii, jj = np.meshgrid(np.arange(Nq), np.arange(Nk), indexing="ij")
    for b in range(B):
        for h in range(H):
            vis = _visible(Nq, Nk, causal, None if key_mask is None else key_mask[b],
                           _block_mask_of(block_mask, b, h), block)
            p, _ = _head_probs(q[b, :, h], k[b, :, h], scale, vis)
            z = dropout_scale(dropout_p, b, h, ii, jj, seed)
            do = dout[b, :, h]
            dv[b, :, h] = (p * z).T @ do
            dp = z * (do @ v[b, :, h].T)
            D = (p * dp).sum(axis=1)
            ds = p * (dp - D[:, None])
            dq[b, :, h] = scale * ds @ k[b, :, h]
            dk[b, :, h] = scale * ds.T @ q[b, :, h]
    return dq, dk, dv
