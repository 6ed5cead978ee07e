"""GPU parity of fa_fwd_masked / fa_bwd_masked (key-padding mask and dropout)
through the C ABI.

Reference: the fp64 oracle's masked attention and dropout (oracle.masked), pinned
on the CPU, with its own Philox4x32-10.  An all-ones mask without dropout must
reproduce the unmasked calls bit for bit, a masked key's dK and dV are exactly
zero, and with V the identity the zeros of O are exactly the dropped (query, key)
pairs, so every keep decision of the kernel is compared with the oracle's.
"""
import numpy as np
import pytest
import torch

from exact_io_aware_54_b200 import fa_bwd, fa_bwd_masked, fa_check, fa_fwd, fa_fwd_masked, synth, workspace
from oracle import masked
from tests._harness import compare_grad, compare_lse, compare_o, default_scale, f64

pytestmark = pytest.mark.gpu


def _run(B, Nq, Nk, H, d, causal, seed, mask_kw, p=0.0, drop_seed=0):
    q, k, v, do = synth.prefill_inputs(seed, B, Nq, Nk, H, d, with_dout=True)
    mask, bits = synth.key_mask_inputs(seed + 7, B, Nk, **mask_kw)
    qc, kc, vc, dc, bc = (t.cuda() for t in (q, k, v, do, bits))
    o, lse = fa_fwd_masked(qc, kc, vc, bc, dropout_p=p, seed=drop_seed, causal=causal)
    dq, dk, dv = fa_bwd_masked(qc, kc, vc, o, dc, lse, bc, dropout_p=p, seed=drop_seed, causal=causal)
    torch.cuda.synchronize()
    assert fa_check(workspace(256, torch.device("cuda"), "fwd")) == 0
    assert fa_check(workspace(256, torch.device("cuda"), "bwd")) == 0
    m = mask.numpy()
    sc = default_scale(d)
    drop = dict(dropout_p=p, seed=drop_seed)
    o_ref, lse_ref = masked.attn_fwd_masked(f64(q), f64(k), f64(v), causal, sc, key_mask=m, **drop)
    compare_o(f64(o), o_ref)
    compare_lse(f64(lse), lse_ref)
    rq, rk, rv = masked.attn_bwd_masked(f64(q), f64(k), f64(v), f64(do), causal, sc, key_mask=m, **drop)
    compare_grad(f64(dq), rq, "dQ")
    compare_grad(f64(dk), rk, "dK")
    compare_grad(f64(dv), rv, "dV")
    # a masked key takes no part: its gradients are exactly zero
    off = ~mask.cuda()
    assert torch.all(dk.permute(0, 2, 1, 3)[off.unsqueeze(1).expand(B, H, Nk)] == 0)
    assert torch.all(dv.permute(0, 2, 1, 3)[off.unsqueeze(1).expand(B, H, Nk)] == 0)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Nq,Nk", [(200, 333), (129, 129), (300, 130)])
def test_random_key_mask(d, causal, Nq, Nk):
    _run(2, Nq, Nk, 3, d, causal, 4000 + Nq + Nk + d, dict(keep=0.6))


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_right_padding_with_an_empty_batch_element(d, causal):
    # batch element 2 has no key at all: its rows get O = 0 and lse = -inf
    _run(3, 256, 384, 2, d, causal, 4100 + d, dict(pad_to=[384, 200, 0]))


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_all_ones_mask_is_the_unmasked_call(d, causal):
    B, N, H = 2, 300, 3
    q, k, v, do = synth.prefill_inputs(4200 + d, B, N, N, H, d, with_dout=True, device="cuda")
    _, bits = synth.key_mask_inputs(0, B, N, pad_to=[N, N])
    bits = bits.cuda()
    o, lse = fa_fwd(q, k, v, causal=causal)
    om, lsem = fa_fwd_masked(q, k, v, bits, causal=causal)
    torch.cuda.synchronize()
    assert torch.equal(o, om) and torch.equal(lse, lsem)
    dq, dk, dv = fa_bwd(q, k, v, o, do, lse, causal=causal)
    dqm, dkm, dvm = fa_bwd_masked(q, k, v, o, do, lse, bits, causal=causal)
    torch.cuda.synchronize()
    assert torch.equal(dk, dkm) and torch.equal(dv, dvm)
    compare_grad(f64(dqm), f64(dq), "dQ masked vs unmasked")  # fp32 atomics: order may differ


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("mask_kw", [dict(keep=0.7), dict(pad_to=[333, 333])])
def test_dropout(d, causal, mask_kw):
    # pad_to = Nk: every key kept, dropout alone
    _run(2, 200, 333, 3, d, causal, 4300 + d + causal, mask_kw, p=0.1, drop_seed=0x123456789)


@pytest.mark.parametrize("d", [64, 128])
def test_dropout_keep_pattern_is_exact(d):
    """V = identity (key j carries e_j): O[i, h, j] = bf16(p_ij z_ij) / l, so O is zero
    exactly where the (query, key) pair was dropped."""
    B, Nq, Nk, H, p, seed = 2, 256, d, 2, 0.25, 99
    q = synth._normal((B, Nq, H, d), 4400, mult=0.1)
    k = synth._normal((B, Nk, H, d), 4401, mult=0.1)  # small scores: no probability underflows
    v = torch.eye(d, dtype=torch.bfloat16)[None, :, None, :].expand(B, Nk, H, d).contiguous()
    o, _ = fa_fwd_masked(q.cuda(), k.cuda(), v.cuda(), None, dropout_p=p, seed=seed)
    torch.cuda.synchronize()
    assert fa_check(workspace(256, torch.device("cuda"), "fwd")) == 0
    ii, hh, jj = np.meshgrid(np.arange(Nq), np.arange(H), np.arange(Nk), indexing="ij")
    for b in range(B):
        kept = masked.dropout_scale(p, b, hh, ii, jj, seed) > 0  # [Nq, H, Nk]
        got = (o[b].float() != 0).cpu().numpy()
        assert np.array_equal(got, kept), f"batch {b}: {int((got != kept).sum())} keep decisions differ"


@pytest.mark.parametrize("d", [64, 128])
def test_zero_dropout_is_the_plain_call(d):
    B, N, H = 2, 300, 3
    q, k, v, do = synth.prefill_inputs(4500 + d, B, N, N, H, d, with_dout=True, device="cuda")
    o, lse = fa_fwd(q, k, v, causal=True)
    om, lsem = fa_fwd_masked(q, k, v, None, dropout_p=0.0, seed=5, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o, om) and torch.equal(lse, lsem)
    dq, dk, dv = fa_bwd(q, k, v, o, do, lse, causal=True)
    dqm, dkm, dvm = fa_bwd_masked(q, k, v, o, do, lse, None, dropout_p=0.0, seed=5, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(dk, dkm) and torch.equal(dv, dvm)
    compare_grad(f64(dqm), f64(dq), "dQ")
