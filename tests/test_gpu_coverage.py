"""Output coverage and out-of-bounds stores, without a memory checker.

Every output buffer is a view into a larger allocation filled with NaN, with a
4 KiB guard band on each side.  After a call, no element of the output may still
be NaN (the call wrote all of it: O, lse, dQ, dK, dV, the decode outputs), and the
guard bands must be bit-for-bit unchanged (no store left the buffer).  Shapes
cover ragged tails, empty causal rows (Nq > Nk) and every head dimension.
"""
import numpy as np
import pytest
import torch

import exact_io_aware_54_b200 as fa
from exact_io_aware_54_b200 import synth

pytestmark = pytest.mark.gpu

GUARD_BYTES = 4096


class Guarded:
    """A NaN-filled buffer with guard bands around the view handed to the call."""

    def __init__(self, shape, dtype):
        self.n = int(np.prod(shape))
        self.g = GUARD_BYTES // torch.tensor([], dtype=dtype).element_size()
        self.base = torch.full((self.g + self.n + self.g,), float("nan"), dtype=dtype, device="cuda")
        self.bits_dtype = torch.int16 if dtype == torch.bfloat16 else torch.int32
        self.nan_bits = self.base[:1].view(self.bits_dtype).clone()
        self.view = self.base[self.g:self.g + self.n].view(shape)

    def check(self, what):
        guards = torch.cat([self.base[:self.g], self.base[self.g + self.n:]]).view(self.bits_dtype)
        assert bool((guards == self.nan_bits).all()), f"{what}: a store reached the guard band"
        assert not bool(torch.isnan(self.view).any()), f"{what}: elements left unwritten"


def _sync_ok(tag):
    torch.cuda.synchronize()
    assert fa.fa_check(fa.workspace(256, torch.device("cuda"), tag)) == 0


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Nq,Nk", [(1, 1), (129, 129), (383, 257), (200, 513)])
def test_forward_and_backward_write_exactly_their_outputs(d, causal, Nq, Nk):
    B, H = 2, 3
    q, k, v, do = synth.prefill_inputs(3000 + Nq + Nk + d, B, Nq, Nk, H, d, with_dout=True, device="cuda")
    o = Guarded((B, Nq, H, d), torch.bfloat16)
    lse = Guarded((B, H, Nq), torch.float32)
    fa.fa_fwd(q, k, v, causal=causal, out=o.view, lse=lse.view)
    _sync_ok("fwd")
    o.check("O")
    lse.check("lse")
    dq = Guarded((B, Nq, H, d), torch.bfloat16)
    dk = Guarded((B, Nk, H, d), torch.bfloat16)
    dv = Guarded((B, Nk, H, d), torch.bfloat16)
    fa.fa_bwd(q, k, v, o.view, do, lse.view, causal=causal, dq=dq.view, dk=dk.view, dv=dv.view)
    _sync_ok("bwd")
    dq.check("dQ")
    dk.check("dK")
    dv.check("dV")


@pytest.mark.parametrize("d", [64, 128])
def test_variable_length_calls_stay_in_their_buffers(d):
    lq = [1, 127, 300, 0, 129]
    lk = [5, 127, 260, 9, 129]
    H = 2
    q = synth._normal((sum(lq), H, d), 3100 + d).cuda()
    k = synth._normal((sum(lk), H, d), 3101 + d).cuda()
    v = synth._normal((sum(lk), H, d), 3102 + d).cuda()
    do = synth._normal((sum(lq), H, d), 3103 + d).cuda()
    cq = torch.tensor(np.concatenate([[0], np.cumsum(lq)]), dtype=torch.int32, device="cuda")
    ck = torch.tensor(np.concatenate([[0], np.cumsum(lk)]), dtype=torch.int32, device="cuda")
    o = Guarded((sum(lq), H, d), torch.bfloat16)
    lse = Guarded((H, sum(lq)), torch.float32)
    fa.fa_fwd_varlen(q, k, v, cq, ck, max(lq), max(lk), causal=True, out=o.view, lse=lse.view)
    _sync_ok("fwd")
    o.check("O")
    lse.check("lse")
    dq = Guarded((sum(lq), H, d), torch.bfloat16)
    dk = Guarded((sum(lk), H, d), torch.bfloat16)
    dv = Guarded((sum(lk), H, d), torch.bfloat16)
    fa.fa_bwd_varlen(q, k, v, o.view, do, lse.view, cq, ck, max(lq), max(lk), causal=True, dq=dq.view, dk=dk.view,
                     dv=dv.view)
    _sync_ok("bwd")
    dq.check("dQ")
    dk.check("dK")
    dv.check("dV")


@pytest.mark.parametrize("d", [64, 128])
def test_decode_writes_exactly_its_outputs(d):
    lengths = [0, 1, 700, 4100]
    B, H = len(lengths), 12
    q, k, v, cu = synth.decode_inputs(3200 + d, lengths, H, d)
    o = Guarded((B, H, d), torch.bfloat16)
    lse = Guarded((B, H), torch.float32)
    fa.fa_decode_splitkv(q.cuda(), k.cuda(), v.cuda(), cu.cuda(), max(lengths), out=o.view, lse=lse.view)
    _sync_ok("decode")
    o.check("O")
    lse.check("lse")
