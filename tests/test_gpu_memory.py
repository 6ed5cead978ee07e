"""Device memory of a long training step is O(N) ("AI Bible 13", section 03,
Theorem 1: the extra memory beyond inputs and outputs grows linearly in N).

At B=1, H=16, N=16384, d=64 one N x N bf16 score matrix of a single head is
512 MiB.  The library allocates nothing itself, so with the outputs and the
workspaces allocated beforehand, the forward and backward calls must add no
allocation at all, and the workspaces (fp32 dQ accumulator, D rows, status word)
stay linear in N, far below one score matrix.
"""
import pytest
import torch

import exact_io_aware_54_b200 as fa
from exact_io_aware_54_b200 import synth

pytestmark = pytest.mark.gpu


def test_long_sequence_step_adds_no_device_memory():
    N, H, d = 16384, 16, 64
    dev = torch.device("cuda", 0)
    q, k, v, do = synth.prefill_inputs(synth.SEEDS["long16k"], 1, N, N, H, d, with_dout=True, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty(1, H, N, dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws_f = fa.workspace(fa.fa_fwd_workspace_size(1, H, N, N, d), dev, "memory_fwd")
    ws_b = fa.workspace(fa.fa_bwd_workspace_size(1, H, N, N, d), dev, "memory_bwd")

    def step():
        fa.fa_fwd(q, k, v, causal=True, out=o, lse=lse, ws=ws_f)
        fa.fa_bwd(q, k, v, o, do, lse, causal=True, dq=dq, dk=dk, dv=dv, ws=ws_b)

    step()  # first launches load the kernels
    torch.cuda.synchronize()
    base = torch.cuda.memory_allocated(dev)
    torch.cuda.reset_peak_memory_stats(dev)
    free0, _ = torch.cuda.mem_get_info(dev)
    step()
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info(dev)
    assert fa.fa_check(ws_f) == 0 and fa.fa_check(ws_b) == 0
    one_score_matrix = N * N * 2
    assert torch.cuda.max_memory_allocated(dev) - base == 0
    assert free0 - free1 < one_score_matrix // 8
    assert ws_f.numel() + ws_b.numel() < one_score_matrix // 4
    assert torch.isfinite(dq.float()).all() and torch.isfinite(dk.float()).all()
