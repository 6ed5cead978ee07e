"""Shared helpers for the GPU parity tests: tolerances and comparisons.

Tolerances (bf16 inputs, fp32 accumulation, N(0,1) data):
  O    : max |o_gpu - o_oracle| <= 1e-2 and mean |.| <= 1e-3
  LSE  : |lse_gpu - lse_oracle| <= 1e-4 * max(1, |lse_oracle|)
  dQ/dK/dV : max |g_gpu - g_oracle| / max(max |g_oracle|, 1e-3) <= 2e-2 (per tensor)
             (the 1e-3 floor only matters when the exact gradient is zero, e.g. a
             single key, where the GPU result is rounding noise of order 1e-7)
"""
import math

import numpy as np
import torch

O_MAX_ABS = 1e-2
O_MEAN_ABS = 1e-3
LSE_REL = 1e-4
GRAD_REL = 2e-2
GRAD_FLOOR = 1e-3


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def compare_o(o_gpu, o_ref, what="O", mean_tol=O_MEAN_ABS, max_tol=O_MAX_ABS):
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    assert o_gpu.shape == o_ref.shape, (o_gpu.shape, o_ref.shape)
    assert np.all(np.isfinite(o_gpu)), f"{what}: non-finite values"
    err = np.abs(o_gpu - o_ref)
    mx, mean = float(err.max(initial=0.0)), float(err.mean()) if err.size else 0.0
    assert mx <= max_tol, f"{what}: max abs err {mx:.3e} > {max_tol}"
    assert mean <= mean_tol, f"{what}: mean abs err {mean:.3e} > {mean_tol}"
    return mx, mean


def compare_lse(lse_gpu, lse_ref, what="LSE"):
    lse_gpu = np.asarray(lse_gpu, dtype=np.float64)
    lse_ref = np.asarray(lse_ref, dtype=np.float64)
    assert lse_gpu.shape == lse_ref.shape
    inf_ref = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse_gpu), inf_ref), f"{what}: -inf rows differ"
    fin = ~inf_ref
    if fin.any():
        err = np.abs(lse_gpu[fin] - lse_ref[fin]) / np.maximum(1.0, np.abs(lse_ref[fin]))
        assert np.all(np.isfinite(lse_gpu[fin])), f"{what}: non-finite"
        assert float(err.max()) <= LSE_REL, f"{what}: rel err {float(err.max()):.3e} > {LSE_REL}"


def compare_grad(g_gpu, g_ref, what):
    g_gpu = np.asarray(g_gpu, dtype=np.float64)
    g_ref = np.asarray(g_ref, dtype=np.float64)
    assert np.all(np.isfinite(g_gpu)), f"{what}: non-finite values"
    scale = max(float(np.abs(g_ref).max(initial=0.0)), GRAD_FLOOR)
    err = float(np.abs(g_gpu - g_ref).max(initial=0.0))
    assert err / scale <= GRAD_REL, f"{what}: normalised max err {err / scale:.3e} > {GRAD_REL}"
    return err / scale


def rounding_floor(o_ref):
    """mean |bf16(o) - o|: the error that storing the exact output in bf16 alone makes."""
    t = torch.from_numpy(np.asarray(o_ref, dtype=np.float64))
    return float((t.to(torch.bfloat16).to(torch.float64) - t).abs().mean())


def default_scale(d):
    return 1.0 / math.sqrt(d)


class OAccumulator:
    """O compared over a whole tensor that is checked slice by slice: the maximum and
    the mean of |o_gpu - o_oracle| are taken over every element of every slice."""

    def __init__(self, what="O"):
        self.what, self.max, self.sum, self.n = what, 0.0, 0.0, 0

    def add(self, o_gpu, o_ref):
        o_gpu = np.asarray(o_gpu, dtype=np.float64)
        o_ref = np.asarray(o_ref, dtype=np.float64)
        assert o_gpu.shape == o_ref.shape, (o_gpu.shape, o_ref.shape)
        assert np.all(np.isfinite(o_gpu)), f"{self.what}: non-finite values"
        err = np.abs(o_gpu - o_ref)
        self.max = max(self.max, float(err.max(initial=0.0)))
        self.sum += float(err.sum())
        self.n += err.size

    def check(self, mean_tol=O_MEAN_ABS, max_tol=O_MAX_ABS):
        mean = self.sum / max(self.n, 1)
        assert self.max <= max_tol, f"{self.what}: max abs err {self.max:.3e} > {max_tol}"
        assert mean <= mean_tol, f"{self.what}: mean abs err {mean:.3e} > {mean_tol}"
        return self.max, mean


class GradAccumulator:
    """One gradient tensor compared slice by slice: max |g_gpu - g_oracle| over the
    whole tensor, normalised by max |g_oracle| over the whole tensor."""

    def __init__(self, what):
        self.what, self.err, self.scale, self.n = what, 0.0, 0.0, 0

    def add(self, g_gpu, g_ref):
        g_gpu = np.asarray(g_gpu, dtype=np.float64)
        g_ref = np.asarray(g_ref, dtype=np.float64)
        assert g_gpu.shape == g_ref.shape, (g_gpu.shape, g_ref.shape)
        assert np.all(np.isfinite(g_gpu)), f"{self.what}: non-finite values"
        self.err = max(self.err, float(np.abs(g_gpu - g_ref).max(initial=0.0)))
        self.scale = max(self.scale, float(np.abs(g_ref).max(initial=0.0)))
        self.n += g_gpu.size

    def check(self):
        rel = self.err / max(self.scale, GRAD_FLOOR)
        assert rel <= GRAD_REL, f"{self.what}: normalised max err {rel:.3e} > {GRAD_REL}"
        return rel


def compare_reordered(o_a, o_b, lse_a, lse_b, what="O"):
    """Two GPU results of the same attention that differ only in the order of their
    fp32 sums (the split-KV decode hands key chunks to CTAs as they become free, so
    which keys share a partial state changes from call to call): O agrees to one
    bf16 step (a bf16 value in [2^e, 2^(e+1)) has steps of 2^(e-7), at most 2^-7 of
    its magnitude) and LSE to 1e-5 relative."""
    a = np.asarray(o_a, dtype=np.float64)
    b = np.asarray(o_b, dtype=np.float64)
    assert a.shape == b.shape
    tol = 2.0 ** -7 * np.maximum(np.abs(a), np.abs(b)) + 1e-6
    bad = np.abs(a - b) > tol
    assert not bad.any(), f"{what}: {int(bad.sum())} elements differ by more than one bf16 step"
    la = np.asarray(lse_a, dtype=np.float64)
    lb = np.asarray(lse_b, dtype=np.float64)
    assert np.array_equal(np.isneginf(la), np.isneginf(lb)), f"LSE of {what}: -inf rows differ"
    fin = np.isfinite(la)
    if fin.any():
        assert float(np.max(np.abs(la[fin] - lb[fin]) / np.maximum(1.0, np.abs(la[fin])))) <= 1e-5
