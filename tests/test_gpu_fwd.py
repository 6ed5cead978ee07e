"""GPU parity of fa_fwd against the fp64 oracle (through the C ABI binding)."""
import pytest
import torch

import oracle
from exact_io_aware_54_b200 import fa_check, fa_fwd, synth, workspace
from tests._harness import OAccumulator, compare_lse, compare_o, default_scale, f64, rounding_floor

pytestmark = pytest.mark.gpu


def _run(q, k, v, causal, scale=None):
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o, lse = fa_fwd(qd, kd, vd, causal=causal, softmax_scale=scale)
    torch.cuda.synchronize()
    assert fa_check(workspace(256, qd.device, "fwd")) == 0
    return o, lse


def _full_check(B, Nq, Nk, H, d, causal, seed, q_mult=1.0, scale=None):
    q, k, v = synth.prefill_inputs(seed, B, Nq, Nk, H, d, q_mult=q_mult)
    sc = default_scale(d) if scale is None else scale
    o, lse = _run(q, k, v, causal, scale)
    o_ref, lse_ref = oracle.attn_fwd(f64(q), f64(k), f64(v), causal, sc)
    mx, mean = compare_o(f64(o), o_ref)
    compare_lse(f64(lse), lse_ref)
    return mx, mean, o_ref


def test_tiny_config_noncausal():
    """B=1, H=2, N=256, d=64, non-causal, scale 1/8 (seed 54001)."""
    _full_check(1, 256, 256, 2, 64, False, synth.SEEDS["tiny"])


def test_tiny_config_q_times_40():
    """Same shape with Q x 40: raw scores span about +-1000, exercising max subtraction."""
    mx, mean, o_ref = _full_check(1, 256, 256, 2, 64, False, synth.SEEDS["tiny"], q_mult=40.0)
    floor = rounding_floor(o_ref)
    assert floor < 1e-3  # the bf16 storage floor itself is inside the bar


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_running_max_moves_across_key_tiles(d, causal):
    """Q x 40 over four key tiles: scores with a spread of about 58 in log2 units, so
    a row's reference max moves by more than the lazy-rescale threshold on later key
    tiles and the O accumulator is rescaled in tensor memory (at d = 128 before the
    first half of that tile's P V).  V is scaled by 1/4 (exact in bf16): with nearly
    one-hot rows O is close to single rows of V, and for |O| >= 4 storing O in bf16
    alone can miss the O bound by half a unit in the last place (1.6e-2)."""
    q, k, v = synth.prefill_inputs(6100 + d + int(causal), 1, 512, 512, 2, d, q_mult=40.0)
    v = v * 0.25
    o, lse = _run(q, k, v, causal)
    o_ref, lse_ref = oracle.attn_fwd(f64(q), f64(k), f64(v), causal, default_scale(d))
    compare_o(f64(o), o_ref)
    compare_lse(f64(lse), lse_ref)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Nq,Nk", [(1, 1), (1, 300), (129, 129), (200, 200), (256, 640), (383, 257), (513, 130),
                                   (640, 1000)])
def test_edge_shapes(d, causal, Nq, Nk):
    _full_check(2, Nq, Nk, 3, d, causal, 1000 + Nq + Nk + d + causal)


@pytest.mark.parametrize("d", [64, 128])
def test_many_items_per_cta(d):
    """More (b, h, q-tile pair) items than SMs: each persistent CTA loops over several."""
    _full_check(4, 512, 512, 48, d, True, 777 + d)


@pytest.mark.parametrize("causal", [False, True])
def test_absent_last_tile_with_many_items_per_cta(causal):
    """Nq % 256 <= 128 leaves the second query tile of the last pair empty; with
    B * H above twice the SM count a persistent CTA meets such items back to back."""
    _full_check(4, 1100, 1100, 80, 64, causal, 888 + causal)


def test_explicit_scale():
    _full_check(1, 300, 300, 2, 64, True, 4242, scale=0.37)


def _whole_tensor_check(B, N, H, d, causal, seed, batch_chunk=None):
    """Every element of O and LSE of the workload against the oracle on the same
    inputs; nothing is subsampled.  The oracle runs on `batch_chunk` batch elements
    at a time (to bound host memory); O's max and mean errors are taken over the
    whole tensor."""
    q, k, v = synth.prefill_inputs(seed, B, N, N, H, d, device="cuda")
    o, lse = fa_fwd(q, k, v, causal=causal)
    torch.cuda.synchronize()
    assert fa_check(workspace(256, q.device, "fwd")) == 0
    acc = OAccumulator()
    step = batch_chunk or B
    for b0 in range(0, B, step):
        sl = slice(b0, min(B, b0 + step))
        o_ref, lse_ref = oracle.attn_fwd(f64(q[sl]), f64(k[sl]), f64(v[sl]), causal, default_scale(d))
        acc.add(f64(o[sl]), o_ref)
        compare_lse(f64(lse[sl]), lse_ref, what=f"LSE[b={b0}..]")
    acc.check()


def test_gpt2_medium_shape_whole_tensor():
    """B=64, H=16, N=1024, d=64, causal (seed 54002): all of O and LSE."""
    _whole_tensor_check(64, 1024, 16, 64, True, synth.SEEDS["gpt2m"], batch_chunk=8)


@pytest.mark.parametrize("causal", [True, False])
def test_long_prefill_whole_tensor(causal):
    """B=1, H=32, N=8192, d=128, causal and non-causal (seed 54003): all of O and LSE."""
    _whole_tensor_check(1, 8192, 32, 128, causal, synth.SEEDS["prefill8k"])


def test_long_sequence_whole_tensor():
    """B=1, H=16, N=16384, d=64, causal (seed 54005): all of O and LSE."""
    _whole_tensor_check(1, 16384, 16, 64, True, synth.SEEDS["long16k"])


def test_deterministic_and_reentrant():
    q, k, v = synth.prefill_inputs(5, 2, 333, 333, 4, 64, device="cuda")
    o1, l1 = fa_fwd(q, k, v, causal=True)
    o2, l2 = fa_fwd(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
