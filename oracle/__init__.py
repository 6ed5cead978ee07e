"""fp64 CPU oracle for exact attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports, loads or calls it, and it shares no code with
that path.

The arithmetic lives in ``oracle.c`` (plain C, fp64, OpenMP over rows/heads);
this module only marshals numpy arrays into it.  See ``oracle.c`` for the
definitions and the passages of the pages they follow:

* "FlashAttention saves IO, not N^2 work", section 1 (S = QK^T/sqrt(d),
  P = softmax(S), O = PV), section 2 (the (m, l, u) state), section 3 (merging
  two block states);
* the Flash Attention wiki note, "Safe Softmax" (max, sum, normalise);
* "AI Bible 13", section 03 (the backward keeps O and the row statistics).

``oracle/masked.py`` (numpy, fp64) adds the key-padding mask and dropout with a
Philox4x32-10 random mask, forward and backward.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_i32p = ctypes.POINTER(ctypes.c_int32)
_i64p = ctypes.POINTER(ctypes.c_int64)


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, -O2, OpenMP).  Returns the path."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            lib.oracle_attn_fwd.argtypes = [_dp, _dp, _dp] + [ctypes.c_int] * 6 + [ctypes.c_double, _dp, _dp]
            lib.oracle_attn_fwd.restype = ctypes.c_int
            lib.oracle_attn_fwd_rows.argtypes = [_dp, _i64p, ctypes.c_int, _dp, _dp] + [ctypes.c_int] * 4 + [
                ctypes.c_double, _dp, _dp]
            lib.oracle_attn_fwd_rows.restype = ctypes.c_int
            lib.oracle_attn_probs.argtypes = [_dp, _dp] + [ctypes.c_int] * 4 + [ctypes.c_double, _dp]
            lib.oracle_attn_probs.restype = ctypes.c_int
            lib.oracle_attn_bwd.argtypes = [_dp] * 4 + [ctypes.c_int] * 6 + [ctypes.c_double, _dp, _dp, _dp]
            lib.oracle_attn_bwd.restype = ctypes.c_int
            lib.oracle_decode.argtypes = [_dp, _dp, _dp, _i32p] + [ctypes.c_int] * 3 + [ctypes.c_double, _dp, _dp]
            lib.oracle_decode.restype = ctypes.c_int
            lib.oracle_row_state.argtypes = [_dp, _dp, ctypes.c_int, ctypes.c_int, _dp, _dp, _dp]
            lib.oracle_row_state.restype = None
            lib.oracle_merge_state.argtypes = [ctypes.c_double, ctypes.c_double, _dp, ctypes.c_double,
                                               ctypes.c_double, _dp, ctypes.c_int, _dp, _dp, _dp]
            lib.oracle_merge_state.restype = None
            lib.oracle_num_threads.argtypes = []
            lib.oracle_num_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray, t=_dp):
    return a.ctypes.data_as(t)


def num_threads() -> int:
    """OpenMP threads the oracle uses (OMP_NUM_THREADS, else all cores)."""
    return int(_load().oracle_num_threads())


def attn_fwd(q, k, v, causal: bool, scale: float):
    """q: [B, Nq, H, d]; k, v: [B, Nk, H, d] -> (o [B, Nq, H, d], lse [B, H, Nq]) in fp64."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Nq, H, d = q.shape
    Nk = k.shape[1]
    assert k.shape == (B, Nk, H, d) and v.shape == (B, Nk, H, d)
    o = np.zeros((B, Nq, H, d))
    lse = np.zeros((B, H, Nq))
    rc = _load().oracle_attn_fwd(_ptr(q), _ptr(k), _ptr(v), B, H, Nq, Nk, d, int(bool(causal)), float(scale),
                                 _ptr(o), _ptr(lse))
    if rc:
        raise MemoryError("oracle_attn_fwd failed")
    return o, lse


def attn_fwd_rows(q_rows, row_idx, k, v, Nq: int, causal: bool, scale: float):
    """Selected query rows of ONE head.  q_rows: [R, d]; row_idx: [R] positions in the
    Nq-row sequence; k, v: [Nk, d].  Returns (o_rows [R, d], lse_rows [R])."""
    q_rows, k, v = _f64(q_rows), _f64(k), _f64(v)
    idx = np.ascontiguousarray(np.asarray(row_idx, dtype=np.int64))
    R, d = q_rows.shape
    Nk = k.shape[0]
    o = np.zeros((R, d))
    lse = np.zeros(R)
    rc = _load().oracle_attn_fwd_rows(_ptr(q_rows), _ptr(idx, _i64p), R, _ptr(k), _ptr(v), int(Nq), Nk, d,
                                      int(bool(causal)), float(scale), _ptr(o), _ptr(lse))
    if rc:
        raise MemoryError("oracle_attn_fwd_rows failed")
    return o, lse


def attn_probs(q, k, causal: bool, scale: float):
    """Probability matrix of ONE head: q [Nq, d], k [Nk, d] -> P [Nq, Nk] (0 where masked)."""
    q, k = _f64(q), _f64(k)
    Nq, d = q.shape
    Nk = k.shape[0]
    P = np.zeros((Nq, Nk))
    if _load().oracle_attn_probs(_ptr(q), _ptr(k), Nq, Nk, d, int(bool(causal)), float(scale), _ptr(P)):
        raise MemoryError("oracle_attn_probs failed")
    return P


def attn_bwd(q, k, v, dout, causal: bool, scale: float):
    """Gradients of sum(O * dout).  Shapes as attn_fwd; returns (dq, dk, dv) in fp64."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, Nq, H, d = q.shape
    Nk = k.shape[1]
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    rc = _load().oracle_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), B, H, Nq, Nk, d, int(bool(causal)),
                                 float(scale), _ptr(dq), _ptr(dk), _ptr(dv))
    if rc:
        raise MemoryError("oracle_attn_bwd failed")
    return dq, dk, dv


def decode(q, k, v, cu_seqlens, scale: float):
    """q: [B, H, d]; k, v: [total, H, d]; cu_seqlens: [B+1] -> (o [B, H, d], lse [B, H])."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
    B, H, d = q.shape
    o = np.zeros((B, H, d))
    lse = np.zeros((B, H))
    if _load().oracle_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(cu, _i32p), B, H, d, float(scale), _ptr(o),
                             _ptr(lse)):
        raise MemoryError("oracle_decode failed")
    return o, lse


def attn_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, causal: bool, scale: float):
    """Forward over packed variable-length sequences: q [total_q, H, d], k, v
    [total_k, H, d], row offsets cu_seqlens_* [B+1] -> (o [total_q, H, d],
    lse [H, total_q]).  Each sequence is one batch element of `attn_fwd` (the
    causal mask bottom-right aligned within it); packing changes nothing else."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    cq = np.asarray(cu_seqlens_q, dtype=np.int64)
    ck = np.asarray(cu_seqlens_k, dtype=np.int64)
    total_q, H, d = q.shape
    o = np.zeros((total_q, H, d))
    lse = np.full((H, total_q), -np.inf)
    for b in range(len(cq) - 1):
        q0, q1, k0, k1 = cq[b], cq[b + 1], ck[b], ck[b + 1]
        if q1 == q0:
            continue
        if k1 == k0:  # no keys: O = 0, lse = -inf
            continue
        ob, lb = attn_fwd(q[None, q0:q1], k[None, k0:k1], v[None, k0:k1], causal, scale)
        o[q0:q1] = ob[0]
        lse[:, q0:q1] = lb[0]
    return o, lse


def attn_bwd_varlen(q, k, v, dout, cu_seqlens_q, cu_seqlens_k, causal: bool, scale: float):
    """Gradients of sum(O * dout) for the packed forward `attn_fwd_varlen`: q, dout
    [total_q, H, d], k, v [total_k, H, d] -> (dq, dk, dv) of the same shapes, fp64.
    Each sequence is one batch element of `attn_bwd`; rows outside every sequence,
    a sequence's queries when it has no keys, and its keys when it has no queries
    get zero gradient (they take no part in the loss)."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    cq = np.asarray(cu_seqlens_q, dtype=np.int64)
    ck = np.asarray(cu_seqlens_k, dtype=np.int64)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(len(cq) - 1):
        q0, q1, k0, k1 = cq[b], cq[b + 1], ck[b], ck[b + 1]
        if q1 == q0 or k1 == k0:
            continue
        g = attn_bwd(q[None, q0:q1], k[None, k0:k1], v[None, k0:k1], dout[None, q0:q1], causal, scale)
        dq[q0:q1], dk[k0:k1], dv[k0:k1] = g[0][0], g[1][0], g[2][0]
    return dq, dk, dv


def decode_paged(q, k_pages, v_pages, block_table, seqlens, scale: float):
    """Decode over a paged cache: key t of sequence b is row t % page_size of page
    block_table[b, t // page_size].  The gathered keys and values of each sequence,
    in key order, go through `decode` (the paging changes where keys live, not what
    is computed)."""
    kp, vp = _f64(k_pages), _f64(v_pages)
    table = np.asarray(block_table, dtype=np.int64)
    lens = np.asarray(seqlens, dtype=np.int64)
    page_size = kp.shape[1]
    ks, vs = [], []
    for b, L in enumerate(lens):
        t = np.arange(int(L))
        pages = table[b, t // page_size]
        assert np.all((pages >= 0) & (pages < kp.shape[0])), "page index outside the cache"
        ks.append(kp[pages, t % page_size])
        vs.append(vp[pages, t % page_size])
    H, d = kp.shape[2], kp.shape[3]
    k = np.concatenate(ks, axis=0) if ks else np.zeros((0, H, d))
    v = np.concatenate(vs, axis=0) if vs else np.zeros((0, H, d))
    cu = np.zeros(len(lens) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(lens)
    return decode(q, k, v, cu, scale)


def row_state(scores, values):
    """(m, l, u) of a stream of scores [n] with values [n, dv] (or [n])."""
    s = _f64(scores).reshape(-1)
    vals = _f64(values)
    scalar = vals.ndim == 1
    dv = 1 if scalar else int(np.prod(vals.shape[1:]))
    vals = vals.reshape(len(s), dv)
    m = ctypes.c_double()
    l = ctypes.c_double()
    u = np.zeros(dv)
    _load().oracle_row_state(_ptr(s), _ptr(np.ascontiguousarray(vals)), len(s), dv, ctypes.byref(m),
                             ctypes.byref(l), _ptr(u))
    return m.value, l.value, (float(u[0]) if scalar else u)


def merge_state(a, b):
    """Merge two (m, l, u) states; u may be a float or a vector."""
    ma, la, ua = a
    mb, lb, ub = b
    scalar = np.ndim(ua) == 0
    ua_, ub_ = _f64(np.atleast_1d(ua)), _f64(np.atleast_1d(ub))
    dv = ua_.shape[0]
    m = ctypes.c_double()
    l = ctypes.c_double()
    u = np.zeros(dv)
    _load().oracle_merge_state(float(ma), float(la), _ptr(ua_), float(mb), float(lb), _ptr(ub_), dv,
                               ctypes.byref(m), ctypes.byref(l), _ptr(u))
    return m.value, l.value, (float(u[0]) if scalar else u)
