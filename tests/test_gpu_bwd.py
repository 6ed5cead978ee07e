"""GPU parity of fa_bwd (with the lse of fa_fwd) against the fp64 oracle's gradients."""
import pytest
import torch

import oracle
from exact_io_aware_54_b200 import fa_bwd, fa_check, fa_fwd, synth, workspace
from tests._harness import GradAccumulator, compare_grad, default_scale, f64

pytestmark = pytest.mark.gpu


def _gpu_grads(q, k, v, do, causal, scale=None):
    o, lse = fa_fwd(q, k, v, causal=causal, softmax_scale=scale)
    dq, dk, dv = fa_bwd(q, k, v, o, do, lse, causal=causal, softmax_scale=scale)
    torch.cuda.synchronize()
    assert fa_check(workspace(256, q.device, "fwd")) == 0
    assert fa_check(workspace(256, q.device, "bwd")) == 0
    return dq, dk, dv


def _full_check(B, Nq, Nk, H, d, causal, seed, scale=None):
    q, k, v, do = synth.prefill_inputs(seed, B, Nq, Nk, H, d, with_dout=True)
    dq, dk, dv = _gpu_grads(q.cuda(), k.cuda(), v.cuda(), do.cuda(), causal, scale)
    sc = default_scale(d) if scale is None else scale
    rq, rk, rv = oracle.attn_bwd(f64(q), f64(k), f64(v), f64(do), causal, sc)
    compare_grad(f64(dq), rq, "dQ")
    compare_grad(f64(dk), rk, "dK")
    compare_grad(f64(dv), rv, "dV")


@pytest.mark.parametrize("causal", [False, True])
def test_tiny_shape(causal):
    _full_check(1, 256, 256, 2, 64, causal, synth.SEEDS["tiny"])


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Nq,Nk", [(1, 1), (1, 200), (129, 129), (200, 200), (256, 640), (383, 257), (513, 130)])
def test_edge_shapes(d, causal, Nq, Nk):
    _full_check(2, Nq, Nk, 3, d, causal, 2000 + Nq + Nk + d + causal)


def test_explicit_scale():
    _full_check(1, 300, 300, 2, 64, True, 99, scale=0.21)


def _whole_tensor_check(B, N, H, d, causal, seed, batch_chunk=None):
    """Every element of dQ, dK and dV against the oracle's gradients on the same
    inputs; nothing is subsampled.  The oracle runs on `batch_chunk` batch elements
    at a time; each gradient's error is normalised by its whole tensor's maximum."""
    q, k, v, do = synth.prefill_inputs(seed, B, N, N, H, d, with_dout=True, device="cuda")
    dq, dk, dv = _gpu_grads(q, k, v, do, causal)
    accs = [GradAccumulator(n) for n in ("dQ", "dK", "dV")]
    step = batch_chunk or B
    for b0 in range(0, B, step):
        sl = slice(b0, min(B, b0 + step))
        refs = oracle.attn_bwd(f64(q[sl]), f64(k[sl]), f64(v[sl]), f64(do[sl]), causal, default_scale(d))
        for acc, g, r in zip(accs, (dq, dk, dv), refs):
            acc.add(f64(g[sl]), r)
    for acc in accs:
        acc.check()


def test_gpt2_medium_shape_whole_tensor():
    """B=64, H=16, N=1024, d=64, causal (seed 54002): all of dQ, dK and dV."""
    _whole_tensor_check(64, 1024, 16, 64, True, synth.SEEDS["gpt2m"], batch_chunk=8)


def test_long_sequence_whole_tensor():
    """B=1, H=16, N=16384, d=64, causal (seed 54005): all of dQ, dK and dV."""
    _whole_tensor_check(1, 16384, 16, 64, True, synth.SEEDS["long16k"])


def test_workspace_reuse_and_determinism_of_dk_dv():
    q, k, v, do = synth.prefill_inputs(7, 2, 500, 500, 4, 64, with_dout=True, device="cuda")
    g1 = _gpu_grads(q, k, v, do, True)
    g2 = _gpu_grads(q, k, v, do, True)
    # dK and dV are reduced inside one CTA in a fixed order; dQ uses fp32 atomics
    assert torch.equal(g1[1], g2[1]) and torch.equal(g1[2], g2[2])
    assert (g1[0].float() - g2[0].float()).abs().max().item() <= 1e-2 * g1[0].float().abs().max().item()
