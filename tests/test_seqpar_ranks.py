"""Sequence-parallel attention's exchange logic on two gloo ranks (CPU).

The library's per-shard attention and merge run on the GPU; here the module's
forward and backward take CPU stand-ins for them (shard attention written out in
numpy, and the oracle's two-block merge rule), so what is tested is the product's
exchange: which shard each rank holds and where it sits in the sequence (the
causal boundary), the all-gather of partial (O, lse) in rank order, the merge of
all of them, and the all-reduce of the partial dQ.  The result must equal the
oracle's attention over the whole sequence, causal or not.
"""
import datetime
import json
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from exact_io_aware_54_b200 import synth


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _visible(Nq, Nk, causal, key_offset, nk_total):
    """[Nq, Nk]: shard key j is visible to query i (bottom-right over the whole sequence)."""
    if not causal:
        return np.ones((Nq, Nk), dtype=bool)
    return (key_offset + np.arange(Nk))[None, :] <= np.arange(Nq)[:, None] + (nk_total - Nq)


def _cpu_attn(scale):
    """Attention over one key shard (the CPU stand-in for the library's call)."""
    def attn(q, k, v, causal, key_offset, nk_total):
        q, k, v = (t.double().numpy() for t in (q, k, v))
        B, Nq, H, d = q.shape
        vis = _visible(Nq, k.shape[1], causal, key_offset, nk_total)
        o, lse = np.zeros_like(q), np.full((B, H, Nq), -np.inf)
        for b in range(B):
            for h in range(H):
                s = np.where(vis, scale * q[b, :, h] @ k[b, :, h].T, -np.inf)
                for i in range(Nq):
                    if not vis[i].any():
                        continue
                    m = s[i].max()
                    p = np.exp(s[i] - m)
                    o[b, i, h] = p @ v[b, :, h] / p.sum()
                    lse[b, h, i] = m + math.log(p.sum())
        return torch.from_numpy(o), torch.from_numpy(lse)
    return attn


def _cpu_merge(o_all, lse_all):
    """The two-block merge rule applied shard by shard (oracle.merge_state)."""
    S, B, Nq, H, d = o_all.shape
    o = np.zeros((B, Nq, H, d))
    lse = np.full((B, H, Nq), -np.inf)
    for b in range(B):
        for h in range(H):
            for i in range(Nq):
                m, l, u = -math.inf, 0.0, np.zeros(d)
                for s in range(S):
                    ls = float(lse_all[s, b, h, i])
                    if ls == -math.inf:
                        continue
                    # a shard's normalised output o_s with l_s = 1 and m_s = lse_s
                    m, l, u = oracle.merge_state((m, l, u), (ls, 1.0, o_all[s, b, i, h].double().numpy()))
                if l > 0:
                    o[b, i, h] = u / l
                    lse[b, h, i] = m + math.log(l)
    return torch.from_numpy(o), torch.from_numpy(lse)


def _cpu_attn_bwd(scale):
    """The backward over one key shard with the merged O and lse (CPU stand-in)."""
    def bwd(q, k, v, o, dout, lse, causal, key_offset, nk_total):
        q, k, v, o, dout, lse = (t.double().numpy() for t in (q, k, v, o, dout, lse))
        B, Nq, H, d = q.shape
        vis = _visible(Nq, k.shape[1], causal, key_offset, nk_total)
        dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
        for b in range(B):
            for h in range(H):
                s = scale * q[b, :, h] @ k[b, :, h].T
                p = np.where(vis, np.exp(s - lse[b, h][:, None]), 0.0)
                dv[b, :, h] = p.T @ dout[b, :, h]
                dp = dout[b, :, h] @ v[b, :, h].T
                D = (dout[b, :, h] * o[b, :, h]).sum(axis=1)
                ds = p * (dp - D[:, None])
                dq[b, :, h] = scale * ds @ k[b, :, h]
                dk[b, :, h] = scale * ds.T @ q[b, :, h]
        return torch.from_numpy(dq), torch.from_numpy(dk), torch.from_numpy(dv)
    return bwd


def _rank_main(rank, world, port, out_dir, causal):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        from exact_io_aware_54_b200 import seqpar
        B, Nq, Nk, H, d, scale = 1, 6, 8, 2, 4, 0.5
        q, k, v, do = (t.double() for t in synth.prefill_inputs(6000, B, Nq, Nk, H, d, with_dout=True))
        shard = Nk // world
        ks, vs = k[:, rank * shard:(rank + 1) * shard], v[:, rank * shard:(rank + 1) * shard]
        o, lse = seqpar.sequence_parallel_fwd(q, ks, vs, causal=causal, attn=_cpu_attn(scale), merge=_cpu_merge)
        dq, dk, dv = seqpar.sequence_parallel_bwd(q, ks, vs, o, do, lse, causal=causal,
                                                  attn_bwd=_cpu_attn_bwd(scale))
        np.save(os.path.join(out_dir, f"r{rank}.npy"),
                np.concatenate([o.numpy().ravel(), lse.numpy().ravel(), dq.numpy().ravel(), dk.numpy().ravel(),
                                dv.numpy().ravel()]))
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
            json.dump({"shapes": [list(t.shape) for t in (o, lse, dq, dk, dv)]}, f)
    finally:
        torch.distributed.destroy_process_group()


@pytest.mark.parametrize("causal", [False, True])
def test_two_ranks_reproduce_whole_sequence_attention(tmp_path, causal):
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path), causal), nprocs=world, join=True)
    B, Nq, Nk, H, d, scale = 1, 6, 8, 2, 4, 0.5
    q, k, v, do = (t.double().numpy() for t in synth.prefill_inputs(6000, B, Nq, Nk, H, d, with_dout=True))
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, causal, scale)
    dq_ref, dk_ref, dv_ref = oracle.attn_bwd(q, k, v, do, causal, scale)
    shard = Nk // world
    for r in range(world):
        flat = np.load(tmp_path / f"r{r}.npy")
        sizes = [o_ref.size, lse_ref.size, dq_ref.size, B * shard * H * d, B * shard * H * d]
        o, lse, dq, dk, dv = np.split(flat, np.cumsum(sizes)[:-1])
        np.testing.assert_allclose(o.reshape(o_ref.shape), o_ref, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(lse.reshape(lse_ref.shape), lse_ref, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(dq.reshape(dq_ref.shape), dq_ref, rtol=1e-10, atol=1e-12)
        sl = slice(r * shard, (r + 1) * shard)
        np.testing.assert_allclose(dk.reshape(B, shard, H, d), dk_ref[:, sl], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(dv.reshape(B, shard, H, d), dv_ref[:, sl], rtol=1e-10, atol=1e-12)
