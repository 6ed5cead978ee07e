"""The bounded-wait failure path on the GPU, without any fault.

fa_selftest_wait_timeout waits, with the library's bounded wait, on a barrier that
nothing arrives on; the wait must give up, record FA_ERR_TIMEOUT in the status
word (read and cleared by fa_check), and leave the context able to run real work.
"""
import pytest
import torch

import oracle
from exact_io_aware_54_b200 import fa_check, fa_fwd, fa_selftest_wait_timeout, synth
from tests._harness import compare_lse, compare_o, default_scale, f64

pytestmark = pytest.mark.gpu

FA_ERR_TIMEOUT = 6


@pytest.mark.parametrize("timeout_us", [50, 2000])
def test_wait_expires_reports_and_context_survives(timeout_us):
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    fa_selftest_wait_timeout(ws, timeout_us)
    assert fa_check(ws) == FA_ERR_TIMEOUT
    assert fa_check(ws) == 0  # the word was cleared
    q, k, v = synth.prefill_inputs(31, 1, 200, 200, 2, 64)
    o, lse = fa_fwd(q.cuda(), k.cuda(), v.cuda(), causal=True)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attn_fwd(f64(q), f64(k), f64(v), True, default_scale(64))
    compare_o(f64(o), o_ref)
    compare_lse(f64(lse), lse_ref)


def test_selftest_argument_checks():
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(Exception):
        fa_selftest_wait_timeout(ws, 0)
    with pytest.raises(Exception):
        fa_selftest_wait_timeout(ws[:8], 100)
