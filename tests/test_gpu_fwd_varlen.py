"""GPU parity of fa_fwd_varlen (packed variable-length forward) through the C ABI.

Reference: the fp64 oracle's variable-length forward.  On a batch of equal
lengths the packed path and the dense fa_fwd run the same tiles in the same
order, so their outputs must agree bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_54_b200 import fa_check, fa_fwd, fa_fwd_varlen, synth, workspace
from tests._harness import compare_lse, compare_o, default_scale, f64

pytestmark = pytest.mark.gpu

FA_ERR_INVALID_ARG = 1


def _inputs(seed, lq, lk, H, d):
    q = synth._normal((sum(lq), H, d), seed)
    k = synth._normal((sum(lk), H, d), seed + 1)
    v = synth._normal((sum(lk), H, d), seed + 2)
    cq = torch.tensor(np.concatenate([[0], np.cumsum(lq)]), dtype=torch.int32)
    ck = torch.tensor(np.concatenate([[0], np.cumsum(lk)]), dtype=torch.int32)
    return q, k, v, cq, ck


def _check(lq, lk, H, d, causal, seed, max_q=None, max_k=None):
    q, k, v, cq, ck = _inputs(seed, lq, lk, H, d)
    mq = max(lq) if max_q is None else max_q
    mk = max(lk) if max_k is None else max_k
    o, lse = fa_fwd_varlen(q.cuda(), k.cuda(), v.cuda(), cq.cuda(), ck.cuda(), mq, mk, causal=causal)
    torch.cuda.synchronize()
    assert fa_check(workspace(256, torch.device("cuda"), "fwd")) == 0
    o_ref, lse_ref = oracle.attn_fwd_varlen(f64(q), f64(k), f64(v), cq.numpy(), ck.numpy(), causal, default_scale(d))
    compare_o(f64(o), o_ref)
    compare_lse(f64(lse), lse_ref)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_ragged_batch(d, causal):
    lq = [1, 127, 128, 129, 300, 513, 64, 1000]
    lk = [1, 200, 128, 129, 300, 130, 700, 1000]
    _check(lq, lk, 3, d, causal, 1100 + d + causal)


@pytest.mark.parametrize("causal", [False, True])
def test_empty_sequences_and_loose_bounds(causal):
    _check([0, 5, 200, 0, 17], [9, 0, 260, 0, 17], 2, 64, causal, 1200 + causal, max_q=400, max_k=600)


def test_many_sequences_over_the_sms():
    rng = np.random.default_rng(1300)
    lq = rng.integers(1, 700, 90).tolist()
    lk = [x + int(rng.integers(0, 200)) for x in lq]
    _check(lq, lk, 8, 64, True, 1300)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_bitwise_equal_to_dense_on_equal_lengths(d, causal):
    B, N, H = 3, 384, 4
    q, k, v = synth.prefill_inputs(1400 + d, B, N, N, H, d)
    o_dense, lse_dense = fa_fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal)
    cu = torch.arange(0, (B + 1) * N, N, dtype=torch.int32)
    o_var, lse_var = fa_fwd_varlen(q.reshape(B * N, H, d).cuda(), k.reshape(B * N, H, d).cuda(),
                                   v.reshape(B * N, H, d).cuda(), cu.cuda(), cu.cuda(), N, N, causal=causal)
    torch.cuda.synchronize()
    assert torch.equal(o_var.reshape(B, N, H, d), o_dense)
    assert torch.equal(lse_var, lse_dense.permute(1, 0, 2).reshape(H, B * N))


def test_offsets_outside_the_buffers_are_reported():
    """cu_seqlens pointing past total_q: that sequence is skipped and recorded
    (fa_check -> FA_ERR_INVALID_ARG); the other sequences are still right."""
    q, k, v, cq, ck = _inputs(1500, [100, 200], [100, 200], 2, 64)
    bad_q = torch.tensor([0, 100, 350], dtype=torch.int32)  # 350 > total_q = 300
    ws = workspace(256, torch.device("cuda"), "fwd")
    o = torch.zeros(300, 2, 64, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(2, 300, dtype=torch.float32, device="cuda")
    fa_fwd_varlen(q.cuda(), k.cuda(), v.cuda(), bad_q.cuda(), ck.cuda(), 250, 200, causal=False, out=o, lse=lse)
    assert fa_check(ws) == FA_ERR_INVALID_ARG
    assert fa_check(ws) == 0
    o_ref, lse_ref = oracle.attn_fwd_varlen(f64(q)[:100], f64(k)[:100], f64(v)[:100], np.array([0, 100]),
                                            np.array([0, 100]), False, default_scale(64))
    compare_o(f64(o)[:100], o_ref)
    compare_lse(f64(lse)[:, :100], lse_ref)


def test_offsets_that_would_wrap_32_bit_arithmetic_are_reported():
    """Sequence 1 ends near 2^31 and sequence 2 starts there and ends at -2^31: both
    are skipped and recorded, and no row outside sequence 0 is written."""
    q, k, v, cq, ck = _inputs(1510, [100, 50, 50], [100, 50, 50], 2, 64)
    bad_q = torch.tensor([0, 100, 2 ** 31 - 5, -2 ** 31], dtype=torch.int32, device="cuda")
    ws = workspace(256, torch.device("cuda"), "fwd")
    assert fa_check(ws) == 0
    o = torch.full((200, 2, 64), 7.0, dtype=torch.bfloat16, device="cuda")
    lse = torch.full((2, 200), 7.0, dtype=torch.float32, device="cuda")
    fa_fwd_varlen(q.cuda(), k.cuda(), v.cuda(), bad_q, ck.cuda(), 150, 100, causal=True, out=o, lse=lse)
    assert fa_check(ws) == FA_ERR_INVALID_ARG
    assert torch.all(o[100:] == 7.0) and torch.all(lse[:, 100:] == 7.0)
    o_ref, lse_ref = oracle.attn_fwd_varlen(f64(q)[:100], f64(k)[:100], f64(v)[:100], np.array([0, 100]),
                                            np.array([0, 100]), True, default_scale(64))
    compare_o(f64(o)[:100], o_ref)
    compare_lse(f64(lse)[:, :100], lse_ref)
