"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module holds random-number generation and nothing of the attention
arithmetic.  Every tensor is drawn in fp32 from N(0, 1) with a seeded
``torch.Generator`` and rounded once to bf16 (round-to-nearest-even); the same
bf16 bits go to the GPU and, widened exactly to fp64, to the CPU oracle.

Prefill tensors are token-major ``[B, N, H, d]``; decode uses ``q [B, H, d]``
and a packed, ragged KV cache ``k, v [total, H, d]`` addressed by
``cu_seqlens [B+1]`` (int32, exclusive prefix sum of the lengths).
"""
from __future__ import annotations

import torch

# seeds of the five workloads (one per workload, tensors drawn Q, K, V, dO with
# seed+0 .. seed+3)
SEEDS = {"tiny": 54001, "gpt2m": 54002, "prefill8k": 54003, "decode": 54004, "long16k": 54005}


def _normal(shape, seed: int, device="cpu", mult: float = 1.0) -> torch.Tensor:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    x = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    if mult != 1.0:
        x.mul_(mult)
    return x.to(torch.bfloat16)


def prefill_inputs(seed: int, B: int, Nq: int, Nk: int, H: int, d: int, q_mult: float = 1.0,
                   with_dout: bool = False, device="cpu"):
    """Q [B, Nq, H, d], K, V [B, Nk, H, d] (and dO [B, Nq, H, d]) as bf16."""
    q = _normal((B, Nq, H, d), seed + 0, device, q_mult)
    k = _normal((B, Nk, H, d), seed + 1, device)
    v = _normal((B, Nk, H, d), seed + 2, device)
    if not with_dout:
        return q, k, v
    do = _normal((B, Nq, H, d), seed + 3, device)
    return q, k, v, do


def ragged_lengths(seed: int, B: int, lo: int, hi: int) -> torch.Tensor:
    """B integer lengths drawn uniformly from [lo, hi] (both ends inclusive)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return torch.randint(lo, hi + 1, (B,), generator=g, dtype=torch.int64)


def cu_seqlens_of(lengths) -> torch.Tensor:
    """Exclusive prefix sum [B+1] as int32 (cu[0] = 0)."""
    lengths = torch.as_tensor(lengths, dtype=torch.int64)
    cu = torch.zeros(len(lengths) + 1, dtype=torch.int64)
    cu[1:] = torch.cumsum(lengths, 0)
    return cu.to(torch.int32)


def decode_inputs(seed: int, lengths, H: int, d: int, device="cpu"):
    """q [B, H, d], packed k, v [sum(lengths), H, d] (bf16) and cu_seqlens [B+1] (int32, CPU)."""
    lengths = torch.as_tensor(lengths, dtype=torch.int64)
    B = len(lengths)
    total = int(lengths.sum())
    cu = cu_seqlens_of(lengths)
    q = _normal((B, H, d), seed + 0, device)
    k = _normal((total, H, d), seed + 1, device)
    v = _normal((total, H, d), seed + 2, device)
    return q, k, v, cu


def paged_decode_inputs(seed: int, lengths, H: int, d: int, page_size: int, spare_pages: int = 3, device="cpu"):
    """A paged KV cache holding the given sequence lengths.

    Returns q [B, H, d], k_pages, v_pages [num_pages, page_size, H, d] (bf16), the
    block table [B, max_pages] and seqlens [B] (int32, CPU).  Pages are handed out
    in a seeded random order (so a sequence's pages are scattered through the
    cache), `spare_pages` pages belong to no sequence, and unused block-table
    entries hold -1.
    """
    lengths = torch.as_tensor(lengths, dtype=torch.int64)
    B = len(lengths)
    pages_per_seq = [(int(L) + page_size - 1) // page_size for L in lengths]
    max_pages = max(1, max(pages_per_seq))
    num_pages = sum(pages_per_seq) + spare_pages
    g = torch.Generator().manual_seed(seed + 3)
    order = torch.randperm(num_pages, generator=g)
    table = torch.full((B, max_pages), -1, dtype=torch.int32)
    nxt = 0
    for b, n in enumerate(pages_per_seq):
        table[b, :n] = order[nxt:nxt + n].to(torch.int32)
        nxt += n
    q = _normal((B, H, d), seed + 0, device)
    k_pages = _normal((num_pages, page_size, H, d), seed + 1, device)
    v_pages = _normal((num_pages, page_size, H, d), seed + 2, device)
    return q, k_pages, v_pages, table, lengths.to(torch.int32)


def key_mask_inputs(seed: int, B: int, Nk: int, keep: float = 0.6, pad_to=None):
    """A key-padding mask: [B, Nk] bool (True = the key takes part) and the same bits
    packed for the library, int32 [B, ceil(Nk / 32)] (bit j % 32 of word j / 32).

    Keys are kept with probability `keep`, drawn from a seeded generator; with
    `pad_to` = [L_0, ..., L_{B-1}] the mask is instead right padding (keys j < L_b
    kept).  The packing is the only transformation: layout, not arithmetic."""
    if pad_to is not None:
        mask = torch.arange(Nk)[None, :] < torch.as_tensor(pad_to, dtype=torch.int64)[:, None]
    else:
        g = torch.Generator(device="cpu")
        g.manual_seed(int(seed))
        mask = torch.rand(B, Nk, generator=g) < keep
    words = (Nk + 31) // 32
    bits = torch.zeros(B, words * 32, dtype=torch.int64)
    bits[:, :Nk] = mask.to(torch.int64)
    weights = (torch.ones(32, dtype=torch.int64) << torch.arange(32, dtype=torch.int64))
    packed = (bits.view(B, words, 32) * weights).sum(-1)
    packed = torch.where(packed >= 2 ** 31, packed - 2 ** 32, packed).to(torch.int32)
    return mask, packed


def block_mask_inputs(seed: int, H: int, Nq: int, Nk: int, keep: float = 0.5, pattern: str = "random"):
    """A block-sparse mask uint8 [H, ceil(Nq / 128), ceil(Nk / 128)] (1 = the block is
    computed).  "random": blocks kept with probability `keep` (seeded); "local": a
    band of the diagonal block and its left neighbour; "strided": every other key
    tile.  Layout only: no attention arithmetic."""
    nq, nk = (Nq + 127) // 128, (Nk + 127) // 128
    if pattern == "random":
        g = torch.Generator(device="cpu")
        g.manual_seed(int(seed))
        m = torch.rand(H, nq, nk, generator=g) < keep
    elif pattern == "local":
        i = torch.arange(nq)[:, None]
        j = torch.arange(nk)[None, :]
        m = ((j == i) | (j == i - 1)).expand(H, nq, nk)
    elif pattern == "strided":
        m = (torch.arange(nk)[None, None, :] % 2 == 0).expand(H, nq, nk)
    else:
        raise ValueError(pattern)
    return m.to(torch.uint8).contiguous()
