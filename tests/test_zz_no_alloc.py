"""The allocation-free decode entry point (fa_decode_splitkv_noalloc).

It serves callers that cannot allocate device memory (an operator whose host
framework owns all device allocations, a serving loop that must not call
cudaMalloc): its chunk states live in the library's own fixed 16 MiB device
array instead of a caller workspace.  Its results must match those of
fa_decode_splitkv on the same inputs, and the fp64 oracle within the decode
tolerances, call after call, since every call reuses the same array.  This file
is collected last on purpose.
"""
import pytest
import torch

import oracle
from exact_io_aware_54_b200 import FAError, fa_decode_num_splits, fa_decode_splitkv, fa_decode_splitkv_noalloc, synth
from tests._harness import compare_lse, compare_o, compare_reordered, default_scale, f64

pytestmark = pytest.mark.gpu

CASES = [([8192], 32, 128), ([1, 100, 3000, 0, 517], 12, 64), ([700, 4096, 33], 20, 128)]

SCRATCH_BYTES = 16 << 20


def _oracle_check(q, k, v, cu, o, lse, d, what):
    o_ref, lse_ref = oracle.decode(f64(q), f64(k), f64(v), cu.cpu().numpy(), default_scale(d))
    compare_o(f64(o), o_ref, what=f"O {what}")
    compare_lse(f64(lse), lse_ref, what=f"LSE {what}")


@pytest.mark.parametrize("case", range(len(CASES)))
def test_noalloc_matches_workspace_entry_point_twice(case):
    lengths, H, d = CASES[case]
    for call in range(2):  # two calls in a row share the scratch array
        q, k, v, cu = synth.decode_inputs(900 + 10 * case + call, lengths, H, d, device="cuda")
        cu = cu.cuda()
        o_ref, lse_ref = fa_decode_splitkv(q, k, v, cu, max(lengths))
        o, lse = fa_decode_splitkv_noalloc(q, k, v, cu, max(lengths))
        torch.cuda.synchronize()
        compare_o(f64(o), f64(o_ref), what=f"O call {call}")
        compare_lse(f64(lse), f64(lse_ref), what=f"LSE call {call}")
        _oracle_check(q, k, v, cu, o, lse, d, f"call {call}")


def test_noalloc_calls_whose_layout_changes():
    """Calls with different B * H in a row: the merge tickets and the chunk states of
    a call land where an earlier call left chunk states or tickets of its own."""
    for i, (lengths, H, d) in enumerate((([900, 50, 3000, 7, 1200], 12, 128), ([4096], 32, 128),
                                         ([300, 17, 1024], 40, 64), ([2000, 5], 8, 128), ([64] * 9, 24, 64))):
        q, k, v, cu = synth.decode_inputs(950 + i, lengths, H, d, device="cuda")
        cu = cu.cuda()
        o, lse = fa_decode_splitkv_noalloc(q, k, v, cu, max(lengths))
        torch.cuda.synchronize()
        _oracle_check(q, k, v, cu, o, lse, d, f"call {i}")


def test_noalloc_at_the_end_of_its_scratch():
    """A shape whose chunk states fill the array to within a few KiB of its end
    (B = 2, H = 32, d = 128, 504 chunk states: 1024 bytes of status word and counters,
    then 504 * 64 * (2 + 128) * 4 bytes of states), twice, against the oracle and the
    workspace entry point with the same split."""
    B, H, d, S = 2, 32, 128, 504
    lengths = [4032, 3001]
    assert fa_decode_num_splits(B, H, max(lengths), d, S) == S
    need = 1024 + S * B * H * (2 + d) * 4
    assert SCRATCH_BYTES - 4096 < need <= SCRATCH_BYTES
    for call in range(2):
        q, k, v, cu = synth.decode_inputs(970 + call, lengths, H, d, device="cuda")
        cu = cu.cuda()
        o, lse = fa_decode_splitkv_noalloc(q, k, v, cu, max(lengths), num_splits=S)
        o_ws, lse_ws = fa_decode_splitkv(q, k, v, cu, max(lengths), num_splits=S)
        torch.cuda.synchronize()
        compare_reordered(f64(o), f64(o_ws), f64(lse), f64(lse_ws))
        _oracle_check(q, k, v, cu, o, lse, d, f"call {call}")
    # one chunk more no longer fits
    assert fa_decode_num_splits(B, H, 4040, d, S + 1) == S + 1
    q, k, v, cu = synth.decode_inputs(975, [4040, 10], H, d, device="cuda")
    with pytest.raises(FAError) as e:
        fa_decode_splitkv_noalloc(q, k, v, cu.cuda(), 4040, num_splits=S + 1)
    assert e.value.status == 4  # FA_ERR_WORKSPACE


def test_noalloc_rejects_shapes_beyond_its_scratch():
    q, k, v, cu = synth.decode_inputs(5, [64] * 64, 32, 128, device="cuda")
    with pytest.raises(FAError) as e:
        fa_decode_splitkv_noalloc(q, k, v, cu.cuda(), 1 << 20, num_splits=4096)
    assert e.value.status == 4  # FA_ERR_WORKSPACE
