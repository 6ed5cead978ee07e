"""GPU parity of fa_bwd_varlen (packed variable-length backward) through the C ABI.

Reference: the fp64 oracle's variable-length backward, compared sequence by
sequence (so a small sequence cannot hide behind a large one's scale).  On a batch
of equal lengths the packed and the dense backward compute every key row's dK and
dV with the same tiles in the same order, so those agree bit for bit; dQ is summed
with fp32 atomics in an order that may differ.
"""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_54_b200 import fa_bwd, fa_bwd_varlen, fa_check, fa_fwd, fa_fwd_varlen, synth, workspace
from tests._harness import compare_grad, default_scale, f64

pytestmark = pytest.mark.gpu

FA_ERR_INVALID_ARG = 1


def _offsets(lengths):
    return torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32)


def _inputs(seed, lq, lk, H, d, extra_q=0, extra_k=0):
    """Packed q, k, v, dO with `extra_*` trailing rows that belong to no sequence."""
    tq, tk = sum(lq) + extra_q, sum(lk) + extra_k
    q = synth._normal((tq, H, d), seed)
    k = synth._normal((tk, H, d), seed + 1)
    v = synth._normal((tk, H, d), seed + 2)
    do = synth._normal((tq, H, d), seed + 3)
    return q, k, v, do, _offsets(lq), _offsets(lk)


def _run(q, k, v, do, cq, ck, mq, mk, causal, sentinel=None):
    qc, kc, vc, dc = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = fa_fwd_varlen(qc, kc, vc, cq.cuda(), ck.cuda(), mq, mk, causal=causal)
    grads = [None, None, None]
    if sentinel is not None:  # pre-filled outputs show which rows the call writes
        grads = [torch.full_like(qc, sentinel), torch.full_like(kc, sentinel), torch.full_like(vc, sentinel)]
    dq, dk, dv = fa_bwd_varlen(qc, kc, vc, o, dc, lse, cq.cuda(), ck.cuda(), mq, mk, causal=causal, dq=grads[0],
                               dk=grads[1], dv=grads[2])
    torch.cuda.synchronize()
    assert fa_check(workspace(256, torch.device("cuda"), "fwd")) == 0
    assert fa_check(workspace(256, torch.device("cuda"), "bwd")) == 0
    return dq, dk, dv


def _compare_per_sequence(dq, dk, dv, ref, cq, ck):
    rq, rk, rv = ref
    for b in range(len(cq) - 1):
        q0, q1, k0, k1 = int(cq[b]), int(cq[b + 1]), int(ck[b]), int(ck[b + 1])
        if q1 > q0:
            compare_grad(f64(dq[q0:q1]), rq[q0:q1], f"dQ[seq {b}]")
        if k1 > k0:
            compare_grad(f64(dk[k0:k1]), rk[k0:k1], f"dK[seq {b}]")
            compare_grad(f64(dv[k0:k1]), rv[k0:k1], f"dV[seq {b}]")


def _check(lq, lk, H, d, causal, seed, max_q=None, max_k=None):
    q, k, v, do, cq, ck = _inputs(seed, lq, lk, H, d)
    mq = max(lq) if max_q is None else max_q
    mk = max(lk) if max_k is None else max_k
    dq, dk, dv = _run(q, k, v, do, cq, ck, mq, mk, causal)
    ref = oracle.attn_bwd_varlen(f64(q), f64(k), f64(v), f64(do), cq.numpy(), ck.numpy(), causal, default_scale(d))
    _compare_per_sequence(dq, dk, dv, ref, cq, ck)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_ragged_batch(d, causal):
    lq = [1, 127, 128, 129, 300, 513, 64, 1000]
    lk = [1, 200, 128, 129, 300, 130, 700, 1000]
    _check(lq, lk, 3, d, causal, 1600 + d + causal)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_empty_sequences_loose_bounds_and_unowned_rows(d, causal):
    """Sequence 0 has keys and no queries (dK = dV = 0), sequence 1 queries and no
    keys (dQ = 0), sequence 3 neither; the buffers end with rows of no sequence:
    dQ is zero there and dK / dV are left as they were."""
    lq, lk = [0, 5, 200, 0, 17], [9, 0, 260, 0, 17]
    q, k, v, do, cq, ck = _inputs(1700 + d + causal, lq, lk, 2, d, extra_q=40, extra_k=150)
    dq, dk, dv = _run(q, k, v, do, cq, ck, 400, 600, causal, sentinel=3.0)
    ref = oracle.attn_bwd_varlen(f64(q), f64(k), f64(v), f64(do), cq.numpy(), ck.numpy(), causal, default_scale(d))
    _compare_per_sequence(dq, dk, dv, ref, cq, ck)
    assert torch.all(dk[0:9] == 0) and torch.all(dv[0:9] == 0)
    assert torch.all(dq[0:5] == 0)
    tq, tk = sum(lq), sum(lk)
    assert torch.all(dq[tq:] == 0)
    assert torch.all(dk[tk:] == 3.0) and torch.all(dv[tk:] == 3.0)


@pytest.mark.parametrize("d", [64, 128])
def test_many_sequences_over_the_sms(d):
    rng = np.random.default_rng(1800 + d)
    lq = rng.integers(1, 700, 90).tolist()
    lk = [x + int(rng.integers(0, 200)) for x in lq]
    _check(lq, lk, 8, d, True, 1800 + d)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [384, 300])
def test_matches_dense_on_equal_lengths(d, causal, N):
    B, H = 3, 4
    q, k, v, do = synth.prefill_inputs(1900 + d + N, B, N, N, H, d, with_dout=True, device="cuda")
    o, lse = fa_fwd(q, k, v, causal=causal)
    dq_d, dk_d, dv_d = fa_bwd(q, k, v, o, do, lse, causal=causal)
    cu = torch.arange(0, (B + 1) * N, N, dtype=torch.int32, device="cuda")
    flat = lambda t: t.reshape(B * N, H, d)
    o_v, lse_v = fa_fwd_varlen(flat(q), flat(k), flat(v), cu, cu, N, N, causal=causal)
    dq_v, dk_v, dv_v = fa_bwd_varlen(flat(q), flat(k), flat(v), o_v, flat(do), lse_v, cu, cu, N, N, causal=causal)
    torch.cuda.synchronize()
    assert fa_check(workspace(256, torch.device("cuda"), "bwd")) == 0
    assert torch.equal(dk_v.reshape(B, N, H, d), dk_d)
    assert torch.equal(dv_v.reshape(B, N, H, d), dv_d)
    compare_grad(f64(dq_v.reshape(B, N, H, d)), f64(dq_d), "dQ packed vs dense")


@pytest.mark.parametrize("d", [64, 128])
def test_offsets_outside_the_buffers_are_reported(d):
    """cu_seqlens_q pointing past total_q: that sequence is skipped and recorded
    (fa_check -> FA_ERR_INVALID_ARG); the other sequence's gradients are right."""
    q, k, v, do, cq, ck = _inputs(2000 + d, [100, 200], [100, 200], 2, d)
    qc, kc, vc, dc = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = fa_fwd_varlen(qc, kc, vc, cq.cuda(), ck.cuda(), 200, 200, causal=True)
    torch.cuda.synchronize()
    ws = workspace(256, torch.device("cuda"), "bwd")
    assert fa_check(ws) == 0
    bad_q = torch.tensor([0, 100, 350], dtype=torch.int32, device="cuda")  # 350 > total_q = 300
    dq, dk, dv = fa_bwd_varlen(qc, kc, vc, o, dc, lse, bad_q, ck.cuda(), 250, 200, causal=True)
    assert fa_check(ws) == FA_ERR_INVALID_ARG
    assert fa_check(ws) == 0
    rq, rk, rv = oracle.attn_bwd_varlen(f64(q)[:100], f64(k)[:100], f64(v)[:100], f64(do)[:100], np.array([0, 100]),
                                        np.array([0, 100]), True, default_scale(d))
    compare_grad(f64(dq[:100]), rq, "dQ[seq 0]")
    compare_grad(f64(dk[:100]), rk, "dK[seq 0]")
    compare_grad(f64(dv[:100]), rv, "dV[seq 0]")


@pytest.mark.parametrize("d", [64, 128])
def test_offsets_that_would_wrap_32_bit_arithmetic_are_reported(d):
    """Key offsets near 2^31 and a negative end: those sequences are skipped and
    recorded; dK / dV rows outside sequence 0 keep their fill."""
    q, k, v, do, cq, ck = _inputs(2100 + d, [100, 50, 50], [100, 50, 50], 2, d)
    qc, kc, vc, dc = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = fa_fwd_varlen(qc, kc, vc, cq.cuda(), ck.cuda(), 100, 100, causal=False)
    torch.cuda.synchronize()
    ws = workspace(256, torch.device("cuda"), "bwd")
    assert fa_check(ws) == 0
    bad_k = torch.tensor([0, 100, 2 ** 31 - 5, -2 ** 31], dtype=torch.int32, device="cuda")
    dk = torch.full_like(kc, 7.0)
    dv = torch.full_like(vc, 7.0)
    dq, dk, dv = fa_bwd_varlen(qc, kc, vc, o, dc, lse, cq.cuda(), bad_k, 100, 150, causal=False, dk=dk, dv=dv)
    assert fa_check(ws) == FA_ERR_INVALID_ARG
    assert torch.all(dk[100:] == 7.0) and torch.all(dv[100:] == 7.0)
    rq, rk, rv = oracle.attn_bwd_varlen(f64(q)[:100], f64(k)[:100], f64(v)[:100], f64(do)[:100], np.array([0, 100]),
                                        np.array([0, 100]), False, default_scale(d))
    compare_grad(f64(dq[:100]), rq, "dQ[seq 0]")
    compare_grad(f64(dk[:100]), rk, "dK[seq 0]")
    compare_grad(f64(dv[:100]), rv, "dV[seq 0]")
