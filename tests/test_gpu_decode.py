"""GPU parity of fa_decode_splitkv against the fp64 oracle (through the C ABI binding)."""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_54_b200 import (fa_check, fa_decode_num_splits, fa_decode_splitkv, fa_decode_splitkv_checked,
                                    fa_decode_workspace_size, synth, workspace)
from tests._harness import OAccumulator, compare_lse, compare_o, compare_reordered, default_scale, f64

pytestmark = pytest.mark.gpu


def _check(lengths, H, d, seed, num_splits=0, max_seqlen=None):
    q, k, v, cu = synth.decode_inputs(seed, lengths, H, d)
    maxL = max(lengths) if max_seqlen is None else max_seqlen
    o, lse = fa_decode_splitkv(q.cuda(), k.cuda(), v.cuda(), cu.cuda(), maxL, num_splits=num_splits)
    torch.cuda.synchronize()
    assert fa_check(workspace(256, torch.device("cuda"), "decode")) == 0
    o_ref, lse_ref = oracle.decode(f64(q), f64(k), f64(v), cu.numpy(), default_scale(d))
    compare_o(f64(o), o_ref)
    compare_lse(f64(lse), lse_ref)


def test_single_request_8k():
    """q_len 1, KV length 8192, H=32, d=128 (seed 54004)."""
    _check([8192], 32, 128, synth.SEEDS["decode"])


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("num_splits", [0, 1, 3, 64])
def test_ragged_small(d, num_splits):
    _check([1, 7, 8, 9, 130, 513, 1000, 2048], 8, d, 91 + d, num_splits=num_splits)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("H", [1, 5, 8, 12, 40])
def test_head_groups(H, d):
    """Head counts of every residue: at d = 64 a CTA serves two heads, so odd H leaves
    a group of one."""
    _check([300, 17, 1024], H, d, 300 + H + d)


def test_empty_and_short_sequences():
    _check([0, 1, 0, 5], 4, 64, 17)


def test_max_seqlen_upper_bound():
    """max_seqlen_k may exceed every actual length."""
    _check([100, 900], 8, 128, 23, max_seqlen=4096)


def test_repeated_calls_reuse_workspace():
    """Merge tickets reset themselves: many calls on one workspace stay correct."""
    for i in range(4):
        _check([777, 3000, 64], 16, 128, 500 + i)


def test_workspace_reuse_across_shapes():
    """One workspace reused by calls whose partial-state layout differs (the merge
    tickets of a later call land where an earlier call kept partial states)."""
    ws = torch.zeros(1 << 24, dtype=torch.uint8, device="cuda")
    for lengths, H in (([900, 50], 12), ([300, 17, 1024], 40), ([64], 3), ([2000, 5, 700, 1], 24)):
        q, k, v, cu = synth.decode_inputs(len(lengths) + H, lengths, H, 128)
        o, lse = fa_decode_splitkv(q.cuda(), k.cuda(), v.cuda(), cu.cuda(), max(lengths), ws=ws)
        torch.cuda.synchronize()
        assert fa_check(ws) == 0
        o_ref, lse_ref = oracle.decode(f64(q), f64(k), f64(v), cu.numpy(), default_scale(128))
        compare_o(f64(o), o_ref)
        compare_lse(f64(lse), lse_ref)


def test_batched_ragged_whole_tensor():
    """64 sequences, H=32, d=128, lengths uniform in [512, 16384] (seed 54004), packed
    with cu_seqlens: every sequence's O and LSE against the oracle (nothing is
    subsampled; the oracle takes one sequence at a time to bound host memory)."""
    seed = synth.SEEDS["decode"]
    lengths = synth.ragged_lengths(seed, 64, 512, 16384)
    q, k, v, cu = synth.decode_inputs(seed, lengths, 32, 128, device="cuda")
    cu_d = cu.cuda()
    o, lse = fa_decode_splitkv(q, k, v, cu_d, int(lengths.max()))
    torch.cuda.synchronize()
    assert fa_check(workspace(256, q.device, "decode")) == 0
    acc = OAccumulator()
    for b in range(64):
        s, e = int(cu[b]), int(cu[b + 1])
        one = np.array([0, e - s], dtype=np.int32)
        o_ref, lse_ref = oracle.decode(f64(q[b:b + 1]), f64(k[s:e]), f64(v[s:e]), one, default_scale(128))
        acc.add(f64(o[b:b + 1]), o_ref)
        compare_lse(f64(lse[b:b + 1]), lse_ref, what=f"LSE[b={b}]")
    acc.check()


def test_checked_equals_unchecked_on_valid_offsets():
    """fa_decode_splitkv_checked computes what fa_decode_splitkv does when the offsets
    fit the buffers (same kernel and plan; the sums agree up to their order)."""
    q, k, v, cu = synth.decode_inputs(61, [300, 17, 1024, 0, 513], 12, 128, device="cuda")
    cu = cu.cuda()
    o1, l1 = fa_decode_splitkv(q, k, v, cu, 1024)
    o2, l2 = fa_decode_splitkv_checked(q, k, v, cu, 1024)
    torch.cuda.synchronize()
    assert fa_check(workspace(256, q.device, "decode")) == 0
    compare_reordered(f64(o1), f64(o2), f64(l1), f64(l2))


@pytest.mark.parametrize("cu_bad,bad", [([0, 200, 500, 900, 650], {2, 3}),     # end past total, end < start
                                        ([-8, 200, 500, 600, 650], {0}),        # negative start
                                        ([0, 200, 500, 600, 651], {3})])        # one row past the end
def test_checked_skips_sequences_outside_the_buffers(cu_bad, bad):
    """Offsets that do not fit k and v: the checked decode skips those sequences before
    any of their rows is read (their o and lse stay as they were, NaN here), computes
    the others as usual and reports FA_ERR_INVALID_ARG through fa_check.  K and V
    are views at the start of larger allocations, so that even a read past total_kv
    could only reach memory this test owns; it must not happen all the same."""
    H, d, T = 8, 128, 650
    B = len(cu_bad) - 1
    _, k_all, v_all, _ = synth.decode_inputs(71, [T + 512], H, d, device="cuda")
    q = synth.decode_inputs(81, [1] * B, H, d, device="cuda")[0]  # seeds 81.. share no draw with k, v
    k, v = k_all[:T], v_all[:T]
    cu = torch.tensor(cu_bad, dtype=torch.int32, device="cuda")
    o = torch.full((B, H, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, H), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.zeros(fa_decode_workspace_size(B, H, 512, d), dtype=torch.uint8, device="cuda")
    fa_decode_splitkv_checked(q, k, v, cu, 512, out=o, lse=lse, ws=ws)
    torch.cuda.synchronize()
    assert fa_check(ws) == 1  # FA_ERR_INVALID_ARG
    for b in range(B):
        if b in bad:
            assert bool(torch.isnan(o[b]).all()) and bool(torch.isnan(lse[b]).all()), f"sequence {b} was written"
            continue
        s0, e0 = cu_bad[b], cu_bad[b + 1]
        one = np.array([0, e0 - s0], dtype=np.int32)
        o_ref, lse_ref = oracle.decode(f64(q[b:b + 1]), f64(k[s0:e0]), f64(v[s0:e0]), one, default_scale(d))
        compare_o(f64(o[b:b + 1]), o_ref, what=f"O[b={b}]")
        compare_lse(f64(lse[b:b + 1]), lse_ref, what=f"LSE[b={b}]")
    # the workspace stays usable: a valid call afterwards reports no fault
    cu_ok = torch.tensor([0, 200, 500, 600, 650], dtype=torch.int32, device="cuda")
    fa_decode_splitkv_checked(q[:4], k, v, cu_ok, 512, ws=ws)
    assert fa_check(ws) == 0


def test_split_count_query():
    assert fa_decode_num_splits(1, 32, 8192, 128, 0) >= 1
    assert fa_decode_num_splits(4, 8, 1000, 64, 3) == 3
