"""GPU parity of fa_fwd_blocksparse / fa_bwd_blocksparse through the C ABI.

Reference: the fp64 oracle's block-sparse attention (oracle.masked with a block
mask over 128 x 128 blocks), pinned on the CPU.  An all-ones mask must reproduce
the dense calls bit for bit (O, lse, dK, dV; dQ is summed with atomics), and a
query tile whose blocks are all skipped gets O = 0 and lse = -inf, a key tile no
kept block reaches dK = dV = 0.
"""
import numpy as np
import pytest
import torch

from exact_io_aware_54_b200 import (fa_bwd, fa_bwd_blocksparse, fa_check, fa_fwd, fa_fwd_blocksparse, synth,
                                    workspace)
from oracle import masked
from tests._harness import compare_grad, compare_lse, compare_o, default_scale, f64

pytestmark = pytest.mark.gpu


def _run(B, Nq, Nk, H, d, causal, seed, bm):
    q, k, v, do = synth.prefill_inputs(seed, B, Nq, Nk, H, d, with_dout=True)
    qc, kc, vc, dc, bmc = (t.cuda() for t in (q, k, v, do, bm))
    o, lse = fa_fwd_blocksparse(qc, kc, vc, bmc, causal=causal)
    dq, dk, dv = fa_bwd_blocksparse(qc, kc, vc, o, dc, lse, bmc, causal=causal)
    torch.cuda.synchronize()
    assert fa_check(workspace(256, torch.device("cuda"), "fwd")) == 0
    assert fa_check(workspace(256, torch.device("cuda"), "bwd")) == 0
    m = bm.numpy().astype(bool)
    sc = default_scale(d)
    o_ref, lse_ref = masked.attn_fwd_masked(f64(q), f64(k), f64(v), causal, sc, block_mask=m, block=(128, 128))
    compare_o(f64(o), o_ref)
    compare_lse(f64(lse), lse_ref)
    rq, rk, rv = masked.attn_bwd_masked(f64(q), f64(k), f64(v), f64(do), causal, sc, block_mask=m, block=(128, 128))
    compare_grad(f64(dq), rq, "dQ")
    compare_grad(f64(dk), rk, "dK")
    compare_grad(f64(dv), rv, "dV")
    return o, lse, dq, dk, dv, m


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("pattern", ["random", "local", "strided"])
def test_patterns(d, causal, pattern):
    B, Nq, Nk, H = 2, 300, 520, 3
    _run(B, Nq, Nk, H, d, causal, 5000 + d + causal, synth.block_mask_inputs(5100 + d, H, Nq, Nk, pattern=pattern))


@pytest.mark.parametrize("d", [64, 128])
def test_skipped_rows_and_keys(d):
    # head 0: query tile 1 keeps no block; key tile 2 is kept by no query tile
    B, N, H = 1, 384, 2
    bm = torch.ones(H, 3, 3, dtype=torch.uint8)
    bm[0, 1, :] = 0
    bm[0, :, 2] = 0
    o, lse, dq, dk, dv, _ = _run(B, N, N, H, d, False, 5200 + d, bm)
    assert torch.all(o[0, 128:256, 0] == 0) and torch.all(torch.isneginf(lse[0, 0, 128:256]))
    assert torch.all(dq[0, 128:256, 0] == 0)
    assert torch.all(dk[0, 256:384, 0] == 0) and torch.all(dv[0, 256:384, 0] == 0)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_all_ones_mask_is_the_dense_call(d, causal):
    B, N, H = 2, 300, 3
    q, k, v, do = synth.prefill_inputs(5300 + d, B, N, N, H, d, with_dout=True, device="cuda")
    bm = torch.ones(H, 3, 3, dtype=torch.uint8, device="cuda")
    o, lse = fa_fwd(q, k, v, causal=causal)
    ob, lseb = fa_fwd_blocksparse(q, k, v, bm, causal=causal)
    torch.cuda.synchronize()
    assert torch.equal(o, ob) and torch.equal(lse, lseb)
    dq, dk, dv = fa_bwd(q, k, v, o, do, lse, causal=causal)
    dqb, dkb, dvb = fa_bwd_blocksparse(q, k, v, o, do, lse, bm, causal=causal)
    torch.cuda.synchronize()
    assert torch.equal(dk, dkb) and torch.equal(dv, dvb)
    compare_grad(f64(dqb), f64(dq), "dQ")
