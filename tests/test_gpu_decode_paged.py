"""GPU parity of fa_decode_paged (split-KV decode over a paged KV cache) through the C ABI.

Reference: the fp64 oracle's paged decode (gather each sequence's keys through its
block table, then the decode definition).  The paged path and the packed path run
the same kernel arithmetic for the same split plan, so on the same keys they agree
up to the order of the fp32 sums (key chunks go to CTAs as they become free).
"""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_54_b200 import fa_check, fa_decode_paged, fa_decode_splitkv, synth, workspace
from tests._harness import compare_lse, compare_o, compare_reordered, default_scale, f64

pytestmark = pytest.mark.gpu

FA_ERR_INVALID_ARG = 1


def _run(lengths, H, d, page_size, seed, num_splits=0, max_seqlen=None):
    q, kp, vp, table, lens = synth.paged_decode_inputs(seed, lengths, H, d, page_size)
    maxL = max(max(lengths), 1) if max_seqlen is None else max_seqlen
    need = -(-maxL // page_size)  # the table must cover max_seqlen_k keys
    if table.shape[1] < need:  # unused entries (-1) past every sequence's pages
        table = torch.cat([table, torch.full((table.shape[0], need - table.shape[1]), -1, dtype=torch.int32)], 1)
    o, lse = fa_decode_paged(q.cuda(), kp.cuda(), vp.cuda(), table.cuda(), lens.cuda(), maxL,
                             num_splits=num_splits)
    torch.cuda.synchronize()
    assert fa_check(workspace(256, torch.device("cuda"), "decode")) == 0
    return (q, kp, vp, table, lens), o, lse


def _check(lengths, H, d, page_size, seed, num_splits=0, max_seqlen=None):
    (q, kp, vp, table, lens), o, lse = _run(lengths, H, d, page_size, seed, num_splits, max_seqlen)
    o_ref, lse_ref = oracle.decode_paged(f64(q), f64(kp), f64(vp), table.numpy(), lens.numpy(), default_scale(d))
    compare_o(f64(o), o_ref)
    compare_lse(f64(lse), lse_ref)


@pytest.mark.parametrize("page_size", [1, 16, 64, 256])
@pytest.mark.parametrize("d", [64, 128])
def test_ragged_pages(page_size, d):
    _check([1, 7, 16, 17, 300, 1000, 2049], 8, d, page_size, 700 + page_size + d)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("H", [1, 5, 12])
def test_head_groups(H, d):
    """Head counts that are not a multiple of the paged kernel's 8-head group."""
    _check([5, 300, 1100], H, d, 16, 900 + H + d)


def test_single_request_8k_pages_of_64():
    """The single-request decode shape (L=8192, H=32, d=128) through 128 scattered pages."""
    _check([8192], 32, 128, 64, synth.SEEDS["decode"])


@pytest.mark.parametrize("H", [1, 5, 12, 40])
def test_head_groups(H):
    _check([300, 17, 1024], H, 128, 16, 800 + H)


@pytest.mark.parametrize("num_splits", [1, 3, 64])
def test_forced_splits(num_splits):
    _check([513, 64, 2000], 8, 64, 32, 900 + num_splits, num_splits=num_splits)


def test_empty_sequences_and_loose_bound():
    _check([0, 5, 0, 130], 4, 64, 16, 17, max_seqlen=1024)


@pytest.mark.parametrize("page_size,d", [(16, 64), (64, 128)])
def test_matches_packed_decode(page_size, d):
    """The same keys, paged and packed, give the same result up to the order of the
    fp32 sums (same plan; chunks go to CTAs as they become free)."""
    lengths = [37, 700, 4096, 1]
    (q, kp, vp, table, lens), o, lse = _run(lengths, 16, d, page_size, 950 + d)
    ks, vs = [], []
    for b, L in enumerate(lengths):
        t = torch.arange(L)
        pages = table[b, t // page_size].long()
        ks.append(kp[pages, t % page_size])
        vs.append(vp[pages, t % page_size])
    k, v = torch.cat(ks), torch.cat(vs)
    cu = torch.zeros(len(lengths) + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(torch.tensor(lengths), 0)
    o2, lse2 = fa_decode_splitkv(q.cuda(), k.cuda(), v.cuda(), cu.cuda(), max(lengths))
    torch.cuda.synchronize()
    compare_reordered(f64(o), f64(o2), f64(lse), f64(lse2))


def test_bad_page_index_is_reported_not_followed():
    """A block-table entry outside the cache is recorded (fa_check -> FA_ERR_INVALID_ARG)
    and replaced by page 0, so no read leaves the cache; a later valid call is fine."""
    q, kp, vp, table, lens = synth.paged_decode_inputs(71, [40, 20], 4, 64, 16)
    bad = table.clone()
    bad[0, 1] = kp.shape[0] + 5  # a page that does not exist, inside the sequence's range
    ws = workspace(256, torch.device("cuda"), "decode")
    fa_decode_paged(q.cuda(), kp.cuda(), vp.cuda(), bad.cuda(), lens.cuda(), 40)
    assert fa_check(ws) == FA_ERR_INVALID_ARG
    assert fa_check(ws) == 0  # the status word was cleared by the read
    _check([40, 20], 4, 64, 16, 71)
