"""The allocation-free decode entry point (fa_decode_splitkv_noalloc).

It serves callers that cannot allocate device memory (an operator whose host
framework owns all device allocations, a serving loop that must not call
cudaMalloc): its chunk states live in the library's own fixed 16 MiB device
array instead of a caller workspace.  Its results must match those of
fa_decode_splitkv on the same inputs, call after call, since every call reuses
the same array.  This file is collected last on purpose.
"""
import pytest
import torch

from exact_io_aware_54_b200 import FAError, fa_decode_splitkv, fa_decode_splitkv_noalloc, synth
from tests._harness import compare_lse, compare_o, f64

pytestmark = pytest.mark.gpu

CASES = [([8192], 32, 128), ([1, 100, 3000, 0, 517], 12, 64), ([700, 4096, 33], 20, 128)]


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


def test_noalloc_rejects_shapes_beyond_its_scratch():
    q, k, v, cu = synth.decode_inputs(5, [64] * 64, 32, 128, device="cuda")
    with pytest.raises(FAError) as e:
        fa_decode_splitkv_noalloc(q, k, v, cu.cuda(), 1 << 20, num_splits=4096)
    assert e.value.status == 4  # FA_ERR_WORKSPACE
