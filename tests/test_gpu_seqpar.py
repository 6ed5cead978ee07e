"""GPU parity of the key-shard merge (fa_merge_partials) and of sequence-parallel
attention emulated on one GPU: the shards run one after another instead of on
separate GPUs, which is the same arithmetic without the exchange (the exchange is
tested on CPU ranks in test_seqpar_ranks.py).

Reference: the fp64 oracle's attention over the whole sequence.
"""
import pytest
import torch

import oracle
from exact_io_aware_54_b200 import (fa_bwd, fa_bwd_shard, fa_check, fa_fwd, fa_fwd_shard, fa_merge_partials, synth,
                                    workspace)
from tests._harness import compare_grad, compare_lse, compare_o, default_scale, f64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("S", [2, 4])
def test_shards_merge_to_whole_sequence_attention(d, S):
    B, Nq, Nk, H = 2, 300, 512, 3
    q, k, v, do = synth.prefill_inputs(6100 + d + S, B, Nq, Nk, H, d, with_dout=True, device="cuda")
    c = Nk // S
    shards = [(k[:, s * c:(s + 1) * c].contiguous(), v[:, s * c:(s + 1) * c].contiguous()) for s in range(S)]
    parts = [fa_fwd(q, ks, vs, causal=False) for ks, vs in shards]
    o, lse = fa_merge_partials(torch.stack([p[0] for p in parts]), torch.stack([p[1] for p in parts]))
    grads = [fa_bwd(q, ks, vs, o, do, lse, causal=False) for ks, vs in shards]
    torch.cuda.synchronize()
    assert fa_check(workspace(256, torch.device("cuda"), "fwd")) == 0
    assert fa_check(workspace(256, torch.device("cuda"), "bwd")) == 0
    sc = default_scale(d)
    o_ref, lse_ref = oracle.attn_fwd(f64(q), f64(k), f64(v), False, sc)
    compare_o(f64(o), o_ref)
    compare_lse(f64(lse), lse_ref)
    dq = sum(g[0].float() for g in grads)
    dk = torch.cat([g[1] for g in grads], dim=1)
    dv = torch.cat([g[2] for g in grads], dim=1)
    rq, rk, rv = oracle.attn_bwd(f64(q), f64(k), f64(v), f64(do), False, sc)
    compare_grad(f64(dq), rq, "dQ")
    compare_grad(f64(dk), rk, "dK")
    compare_grad(f64(dv), rv, "dV")


@pytest.mark.parametrize("d", [64, 128])
def test_shards_without_keys_contribute_nothing(d):
    B, Nq, H = 1, 200, 2
    o_parts = synth._normal((3, B, Nq, H, d), 6200).cuda()
    lse_parts = synth._normal((3, B, H, Nq), 6201).float().cuda()
    lse_parts[1] = -float("inf")                  # shard 1 sees no key at all
    lse_parts[0, :, :, :50] = -float("inf")       # rows 0..49 see keys only in shard 2
    lse_parts[2, :, :, :50] = -float("inf")
    lse_parts[2, :, :, :10] = 5.0                 # ... except rows 0..9
    o, lse = fa_merge_partials(o_parts, lse_parts)
    torch.cuda.synchronize()
    # rows 10..49: no shard has keys
    assert torch.all(o[:, 10:50] == 0) and torch.all(torch.isneginf(lse[:, :, 10:50]))
    # rows 0..9: shard 2 alone, weight exactly 1
    assert torch.equal(o[:, :10], o_parts[2, :, :10]) and torch.equal(lse[:, :, :10], lse_parts[2, :, :, :10])
    # the other rows: shards 0 and 2 by the merge rule
    lp = lse_parts[[0, 2], :, :, 50:].double()
    M = lp.max(dim=0).values
    w = torch.exp(lp - M)
    ref = (w.permute(0, 1, 3, 2)[..., None] * o_parts[[0, 2], :, 50:].double()).sum(0) / w.sum(0).permute(0, 2, 1)[..., None]
    compare_o(f64(o[:, 50:]), ref.cpu().numpy())
    compare_lse(f64(lse[:, :, 50:]), (M + torch.log(w.sum(0))).cpu().numpy())


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("S", [2, 4])
@pytest.mark.parametrize("Nq", [300, 512])
def test_causal_shards_merge_to_whole_sequence_attention(d, S, Nq):
    """Causal shards see the bottom-right boundary of the whole sequence; with
    Nq < Nk the first query rows see no key of the last shards (lse = -inf there)."""
    B, Nk, H = 2, 512, 3
    q, k, v, do = synth.prefill_inputs(6300 + d + S + Nq, B, Nq, Nk, H, d, with_dout=True, device="cuda")
    c = Nk // S
    shards = [(k[:, s * c:(s + 1) * c].contiguous(), v[:, s * c:(s + 1) * c].contiguous()) for s in range(S)]
    parts = [fa_fwd_shard(q, ks, vs, s * c, Nk) for s, (ks, vs) in enumerate(shards)]
    o, lse = fa_merge_partials(torch.stack([p[0] for p in parts]), torch.stack([p[1] for p in parts]))
    grads = [fa_bwd_shard(q, ks, vs, o, do, lse, s * c, Nk) for s, (ks, vs) in enumerate(shards)]
    torch.cuda.synchronize()
    assert fa_check(workspace(256, torch.device("cuda"), "fwd")) == 0
    assert fa_check(workspace(256, torch.device("cuda"), "bwd")) == 0
    sc = default_scale(d)
    o_ref, lse_ref = oracle.attn_fwd(f64(q), f64(k), f64(v), True, sc)
    compare_o(f64(o), o_ref)
    compare_lse(f64(lse), lse_ref)
    dq = sum(g[0].float() for g in grads)
    dk = torch.cat([g[1] for g in grads], dim=1)
    dv = torch.cat([g[2] for g in grads], dim=1)
    rq, rk, rv = oracle.attn_bwd(f64(q), f64(k), f64(v), f64(do), True, sc)
    compare_grad(f64(dq), rq, "dQ")
    compare_grad(f64(dk), rk, "dK")
    compare_grad(f64(dv), rv, "dV")


@pytest.mark.parametrize("d", [64, 128])
def test_one_shard_is_the_whole_causal_call(d):
    B, N, H = 2, 300, 3
    q, k, v, do = synth.prefill_inputs(6400 + d, B, N, N, H, d, with_dout=True, device="cuda")
    o, lse = fa_fwd(q, k, v, causal=True)
    os_, lses = fa_fwd_shard(q, k, v, 0, N)
    torch.cuda.synchronize()
    assert torch.equal(o, os_) and torch.equal(lse, lses)
    dq, dk, dv = fa_bwd(q, k, v, o, do, lse, causal=True)
    dqs, dks, dvs = fa_bwd_shard(q, k, v, o, do, lse, 0, N)
    torch.cuda.synchronize()
    assert torch.equal(dk, dks) and torch.equal(dv, dvs)
    compare_grad(f64(dqs), f64(dq), "dQ")
