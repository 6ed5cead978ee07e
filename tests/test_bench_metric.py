"""The algorithmic work behind every rate bench.py reports, on CPU.

A rate is a work count divided by a measured time, so the counts are pinned here
against a definition they do not share code with: the (query, key) pairs that take
part are counted by building the attention mask element by element (bottom-right
aligned causal mask: query i sees key j iff j <= i + Nk - Nq), and the forward and
backward FLOPs are 2 multiply-adds per pair and head dimension for each matrix
product (2 products forward: Q K^T and P V; 5 backward: the recomputed S, dP, dV,
dK and dQ).
"""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _mask_pairs(Nq, Nk, causal):
    i = np.arange(Nq)[:, None]
    j = np.arange(Nk)[None, :]
    keep = (j <= i + Nk - Nq) if causal else np.ones((Nq, Nk), dtype=bool)
    return int(keep.sum())


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Nq,Nk", [(1, 1), (1, 300), (7, 3), (3, 7), (129, 129), (256, 640), (513, 130), (200, 200)])
def test_pairs_match_the_mask(Nq, Nk, causal):
    assert bench.causal_pairs(Nq, Nk, causal) == _mask_pairs(Nq, Nk, causal)


@pytest.mark.parametrize("causal", [False, True])
def test_flops_are_two_per_multiply_add(causal):
    B, H, N, d = 2, 3, 300, 64
    pairs = _mask_pairs(N, N, causal)
    assert bench.fwd_flops(B, H, N, N, d, causal) == 2 * 2 * B * H * d * pairs
    assert bench.bwd_flops(B, H, N, N, d, causal) == 5 * 2 * B * H * d * pairs


def test_the_workloads_counts():
    # the training step of B=64, H=16, N=1024, d=64, causal: 1024 * 1025 / 2 pairs per head
    assert bench.fwd_flops(64, 16, 1024, 1024, 64, True) == 137_573_171_200
    assert bench.bwd_flops(64, 16, 1024, 1024, 64, True) == 343_932_928_000
    # the 8K prefill of B=1, H=32, d=128, causal and not
    assert bench.fwd_flops(1, 32, 8192, 8192, 128, True) == 4 * 32 * 128 * (8192 * 8193 // 2)
    assert bench.fwd_flops(1, 32, 8192, 8192, 128, False) == 4 * 32 * 128 * 8192 * 8192
    # the 16K training step of B=1, H=16, d=64, causal
    assert bench.fwd_flops(1, 16, 16384, 16384, 64, True) + bench.bwd_flops(1, 16, 16384, 16384, 64, True) == \
        14 * 16 * 64 * (16384 * 16385 // 2)
