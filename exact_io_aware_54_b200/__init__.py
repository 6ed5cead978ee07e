"""Exact, IO-aware multi-head attention for NVIDIA B200 (sm_100a).

Thin Python binding over the C ABI of ``libfa.so`` (declared in ``include/fa.h``):
argument marshalling only.  Every step of the computation runs in the library's
CUDA kernels; PyTorch only provides device memory and the current stream.  There
is no CPU or library fallback: when ``libfa.so`` is missing or cannot be loaded,
every call raises.

Entry points (same names as the C ABI):

* :func:`fa_fwd` -- forward pass, returns ``(o, lse)``;
* :func:`fa_bwd` -- recompute backward pass, returns ``(dq, dk, dv)``;
* :func:`fa_decode_splitkv` -- split-KV decode over a ragged packed KV cache,
  returns ``(o, lse)``;
* :func:`fa_check` -- synchronise and read the kernels' status word.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

__all__ = [
    "FAError", "lib_path", "load", "fa_fwd", "fa_bwd", "fa_fwd_masked", "fa_bwd_masked", "fa_fwd_blocksparse",
    "fa_bwd_blocksparse", "fa_fwd_varlen", "fa_bwd_varlen", "fa_decode_splitkv", "fa_decode_splitkv_noalloc",
    "fa_decode_splitkv_checked", "fa_decode_paged", "fa_merge_partials", "fa_fwd_shard", "fa_bwd_shard", "fa_check",
    "fa_fwd_workspace_size", "fa_bwd_workspace_size",
    "fa_bwd_varlen_workspace_size", "fa_decode_workspace_size", "fa_decode_num_splits",
    "fa_version", "STATUS",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
STATUS = {0: "FA_OK", 1: "FA_ERR_INVALID_ARG", 2: "FA_ERR_UNSUPPORTED", 3: "FA_ERR_ALIGNMENT",
          4: "FA_ERR_WORKSPACE", 5: "FA_ERR_CUDA", 6: "FA_ERR_TIMEOUT"}


class FAError(RuntimeError):
    """A non-zero fa_status returned by the library."""

    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {STATUS.get(status, status)}")
        self.status = status


def lib_path() -> str:
    return os.environ.get("FA_LIB", os.path.join(_HERE, "libfa.so"))


_lib = None
_lock = threading.Lock()
_vp = ctypes.c_void_p
_i = ctypes.c_int
_f = ctypes.c_float
_sz = ctypes.c_size_t


def load():
    """Load libfa.so (raises if it is absent: there is no fallback path)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        path = lib_path()
        if not os.path.exists(path):
            raise ImportError(f"libfa.so not found at {path}; build it with "
                              f"`python -m exact_io_aware_54_b200.build`")
        lib = ctypes.CDLL(path)
        lib.fa_fwd.argtypes = [_vp] * 5 + [_i] * 6 + [_f, _vp, _sz, _vp]
        lib.fa_bwd.argtypes = [_vp] * 9 + [_i] * 6 + [_f, _vp, _sz, _vp]
        lib.fa_decode_splitkv.argtypes = [_vp] * 4 + [_i] * 6 + [_f, _i, _vp, _vp, _vp, _sz, _vp]
        lib.fa_decode_splitkv_noalloc.argtypes = [_vp] * 4 + [_i] * 6 + [_f, _i, _vp, _vp, _vp]
        lib.fa_decode_splitkv_checked.argtypes = [_vp] * 4 + [_i] * 7 + [_f, _i, _vp, _vp, _vp, _sz, _vp]
        lib.fa_decode_paged.argtypes = [_vp] * 5 + [_i] * 7 + [_f, _i, _vp, _vp, _vp, _sz, _vp]
        lib.fa_fwd_varlen.argtypes = [_vp] * 7 + [_i] * 8 + [_f, _vp, _sz, _vp]
        lib.fa_bwd_varlen.argtypes = [_vp] * 11 + [_i] * 8 + [_f, _vp, _sz, _vp]
        _u64 = ctypes.c_ulonglong
        lib.fa_fwd_masked.argtypes = [_vp] * 6 + [_f, _u64] + [_i] * 6 + [_f, _vp, _sz, _vp]
        lib.fa_bwd_masked.argtypes = [_vp] * 10 + [_f, _u64] + [_i] * 6 + [_f, _vp, _sz, _vp]
        lib.fa_fwd_blocksparse.argtypes = [_vp] * 6 + [_i] * 6 + [_f, _vp, _sz, _vp]
        lib.fa_bwd_blocksparse.argtypes = [_vp] * 10 + [_i] * 6 + [_f, _vp, _sz, _vp]
        lib.fa_merge_partials.argtypes = [_vp, _vp] + [_i] * 5 + [_vp, _vp, _vp]
        lib.fa_fwd_shard.argtypes = [_vp] * 5 + [_i] * 7 + [_f, _vp, _sz, _vp]
        lib.fa_bwd_shard.argtypes = [_vp] * 9 + [_i] * 7 + [_f, _vp, _sz, _vp]
        for fn in (lib.fa_fwd, lib.fa_bwd, lib.fa_decode_splitkv, lib.fa_decode_splitkv_noalloc,
                   lib.fa_decode_splitkv_checked, lib.fa_decode_paged, lib.fa_fwd_varlen, lib.fa_bwd_varlen,
                   lib.fa_fwd_masked, lib.fa_bwd_masked, lib.fa_fwd_blocksparse, lib.fa_bwd_blocksparse,
                   lib.fa_merge_partials, lib.fa_fwd_shard, lib.fa_bwd_shard):
            fn.restype = _i
        lib.fa_fwd_workspace_size.argtypes = [_i] * 5
        lib.fa_fwd_workspace_size.restype = _sz
        lib.fa_bwd_workspace_size.argtypes = [_i] * 5
        lib.fa_bwd_workspace_size.restype = _sz
        lib.fa_bwd_varlen_workspace_size.argtypes = [_i] * 3
        lib.fa_bwd_varlen_workspace_size.restype = _sz
        lib.fa_decode_workspace_size.argtypes = [_i] * 5
        lib.fa_decode_workspace_size.restype = _sz
        lib.fa_decode_num_splits.argtypes = [_i] * 5
        lib.fa_decode_num_splits.restype = _i
        lib.fa_selftest_wait_timeout.argtypes = [_vp, _sz, ctypes.c_uint, _vp]
        lib.fa_selftest_wait_timeout.restype = _i
        lib.fa_check.argtypes = [_vp, _vp]
        lib.fa_check.restype = _i
        lib.fa_status_string.argtypes = [_i]
        lib.fa_status_string.restype = ctypes.c_char_p
        lib.fa_version.argtypes = []
        lib.fa_version.restype = ctypes.c_char_p
        _lib = lib
        return lib


def fa_version() -> str:
    return load().fa_version().decode()


def fa_fwd_workspace_size(B, H, Nq, Nk, d) -> int:
    return int(load().fa_fwd_workspace_size(B, H, Nq, Nk, d))


def fa_bwd_workspace_size(B, H, Nq, Nk, d) -> int:
    return int(load().fa_bwd_workspace_size(B, H, Nq, Nk, d))


def fa_bwd_varlen_workspace_size(H, total_q, d) -> int:
    return int(load().fa_bwd_varlen_workspace_size(H, total_q, d))


def fa_decode_workspace_size(B, H, max_seqlen_k, d, num_splits=0) -> int:
    return int(load().fa_decode_workspace_size(B, H, max_seqlen_k, d, num_splits))


def fa_decode_num_splits(B, H, max_seqlen_k, d, num_splits=0) -> int:
    return int(load().fa_decode_num_splits(B, H, max_seqlen_k, d, num_splits))


# --------------------------------------------------------------------------- workspaces

_ws_cache: dict = {}


def workspace(nbytes: int, device, tag: str = "default") -> torch.Tensor:
    """A zero-initialised workspace of at least `nbytes`, reused per (device, tag).

    The library keeps a workspace consistent between calls (tickets reset
    themselves, fa_check clears the status word), so it is zeroed only once."""
    dev = torch.device(device)
    key = (dev.type, dev.index if dev.index is not None else torch.cuda.current_device(), tag)
    ws = _ws_cache.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=dev)
        _ws_cache[key] = ws
    return ws


def _stream_ptr(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _check_tensor(name, t, dtype, shape=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _raise(fn, status):
    if status != 0:
        raise FAError(fn, status)


def _scale(softmax_scale):
    return 0.0 if softmax_scale is None else float(softmax_scale)


# --------------------------------------------------------------------------- entry points


def fa_fwd(q, k, v, causal: bool = False, softmax_scale=None, out=None, lse=None, ws=None):
    """Forward pass.  q [B, Nq, H, d], k/v [B, Nk, H, d] bf16 -> (o [B, Nq, H, d], lse [B, H, Nq] fp32)."""
    lib = load()
    B, Nq, H, d = q.shape
    Nk = k.shape[1]
    _check_tensor("q", q, torch.bfloat16)
    _check_tensor("k", k, torch.bfloat16, (B, Nk, H, d))
    _check_tensor("v", v, torch.bfloat16, (B, Nk, H, d))
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    _check_tensor("out", out, torch.bfloat16, q.shape)
    _check_tensor("lse", lse, torch.float32, (B, H, Nq))
    need = lib.fa_fwd_workspace_size(B, H, Nq, Nk, d)
    if ws is None:
        ws = workspace(need, q.device, "fwd")
    st = lib.fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), B, H, Nq, Nk, d,
                    int(bool(causal)), _scale(softmax_scale), ws.data_ptr(), ws.numel(), _stream_ptr(q.device))
    _raise("fa_fwd", st)
    return out, lse


def _check_key_mask(key_mask, B, Nk):
    _check_tensor("key_mask", key_mask, torch.int32, (B, (Nk + 31) // 32))


def fa_fwd_masked(q, k, v, key_mask=None, dropout_p: float = 0.0, seed: int = 0, causal: bool = False,
                  softmax_scale=None, out=None, lse=None, ws=None):
    """Forward with a key-padding mask and dropout.  key_mask: int32 [B, ceil(Nk / 32)]
    on the device, bit j % 32 of word j / 32 set when key j takes part (see
    synth.key_mask_inputs), or None.  Returns (o, lse) as fa_fwd."""
    lib = load()
    B, Nq, H, d = q.shape
    Nk = k.shape[1]
    _check_tensor("q", q, torch.bfloat16)
    _check_tensor("k", k, torch.bfloat16, (B, Nk, H, d))
    _check_tensor("v", v, torch.bfloat16, (B, Nk, H, d))
    if key_mask is not None:
        _check_key_mask(key_mask, B, Nk)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device) if lse is None else lse
    _check_tensor("out", out, torch.bfloat16, q.shape)
    _check_tensor("lse", lse, torch.float32, (B, H, Nq))
    if ws is None:
        ws = workspace(lib.fa_fwd_workspace_size(B, H, Nq, Nk, d), q.device, "fwd")
    st = lib.fa_fwd_masked(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                           None if key_mask is None else key_mask.data_ptr(), float(dropout_p), int(seed),
                           B, H, Nq, Nk, d, int(bool(causal)), _scale(softmax_scale), ws.data_ptr(), ws.numel(),
                           _stream_ptr(q.device))
    _raise("fa_fwd_masked", st)
    return out, lse


def fa_bwd_masked(q, k, v, o, dout, lse, key_mask=None, dropout_p: float = 0.0, seed: int = 0, causal: bool = False,
                  softmax_scale=None, dq=None, dk=None, dv=None, ws=None):
    """Backward of fa_fwd_masked with the same key_mask, dropout_p and seed.
    Returns (dq, dk, dv) in bf16."""
    lib = load()
    B, Nq, H, d = q.shape
    Nk = k.shape[1]
    for name, t, shp in (("q", q, None), ("k", k, (B, Nk, H, d)), ("v", v, (B, Nk, H, d)), ("o", o, q.shape),
                         ("dout", dout, q.shape)):
        _check_tensor(name, t, torch.bfloat16, shp)
    _check_tensor("lse", lse, torch.float32, (B, H, Nq))
    if key_mask is not None:
        _check_key_mask(key_mask, B, Nk)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if ws is None:
        ws = workspace(lib.fa_bwd_workspace_size(B, H, Nq, Nk, d), q.device, "bwd")
    st = lib.fa_bwd_masked(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dout.data_ptr(), lse.data_ptr(),
                           dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                           None if key_mask is None else key_mask.data_ptr(), float(dropout_p), int(seed), B, H, Nq,
                           Nk, d, int(bool(causal)), _scale(softmax_scale), ws.data_ptr(), ws.numel(),
                           _stream_ptr(q.device))
    _raise("fa_bwd_masked", st)
    return dq, dk, dv


def _check_block_mask(block_mask, H, Nq, Nk):
    _check_tensor("block_mask", block_mask, torch.uint8, (H, (Nq + 127) // 128, (Nk + 127) // 128))


def fa_fwd_blocksparse(q, k, v, block_mask, causal: bool = False, softmax_scale=None, out=None, lse=None, ws=None):
    """Block-sparse forward.  block_mask: uint8 [H, ceil(Nq/128), ceil(Nk/128)] on the
    device (0 skips the block).  Returns (o, lse) as fa_fwd."""
    lib = load()
    B, Nq, H, d = q.shape
    Nk = k.shape[1]
    _check_tensor("q", q, torch.bfloat16)
    _check_tensor("k", k, torch.bfloat16, (B, Nk, H, d))
    _check_tensor("v", v, torch.bfloat16, (B, Nk, H, d))
    _check_block_mask(block_mask, H, Nq, Nk)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device) if lse is None else lse
    _check_tensor("out", out, torch.bfloat16, q.shape)
    _check_tensor("lse", lse, torch.float32, (B, H, Nq))
    if ws is None:
        ws = workspace(lib.fa_fwd_workspace_size(B, H, Nq, Nk, d), q.device, "fwd")
    st = lib.fa_fwd_blocksparse(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                block_mask.data_ptr(), B, H, Nq, Nk, d, int(bool(causal)), _scale(softmax_scale),
                                ws.data_ptr(), ws.numel(), _stream_ptr(q.device))
    _raise("fa_fwd_blocksparse", st)
    return out, lse


def fa_bwd_blocksparse(q, k, v, o, dout, lse, block_mask, causal: bool = False, softmax_scale=None, dq=None,
                       dk=None, dv=None, ws=None):
    """Backward of fa_fwd_blocksparse with the same block_mask.  Returns (dq, dk, dv) in bf16."""
    lib = load()
    B, Nq, H, d = q.shape
    Nk = k.shape[1]
    for name, t, shp in (("q", q, None), ("k", k, (B, Nk, H, d)), ("v", v, (B, Nk, H, d)), ("o", o, q.shape),
                         ("dout", dout, q.shape)):
        _check_tensor(name, t, torch.bfloat16, shp)
    _check_tensor("lse", lse, torch.float32, (B, H, Nq))
    _check_block_mask(block_mask, H, Nq, Nk)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if ws is None:
        ws = workspace(lib.fa_bwd_workspace_size(B, H, Nq, Nk, d), q.device, "bwd")
    st = lib.fa_bwd_blocksparse(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dout.data_ptr(),
                                lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), block_mask.data_ptr(),
                                B, H, Nq, Nk, d, int(bool(causal)), _scale(softmax_scale), ws.data_ptr(), ws.numel(),
                                _stream_ptr(q.device))
    _raise("fa_bwd_blocksparse", st)
    return dq, dk, dv


def fa_fwd_shard(q, k, v, key_offset: int, Nk_total: int, softmax_scale=None, out=None, lse=None, ws=None):
    """Causal attention of all queries q [B, Nq, H, d] over a key shard k, v
    [B, Nk, H, d] holding keys key_offset .. key_offset + Nk - 1 of Nk_total.
    Returns (o, lse) as fa_fwd (rows that see no key of the shard: 0 and -inf)."""
    lib = load()
    B, Nq, H, d = q.shape
    Nk = k.shape[1]
    _check_tensor("q", q, torch.bfloat16)
    _check_tensor("k", k, torch.bfloat16, (B, Nk, H, d))
    _check_tensor("v", v, torch.bfloat16, (B, Nk, H, d))
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device) if lse is None else lse
    _check_tensor("out", out, torch.bfloat16, q.shape)
    _check_tensor("lse", lse, torch.float32, (B, H, Nq))
    if ws is None:
        ws = workspace(lib.fa_fwd_workspace_size(B, H, Nq, Nk, d), q.device, "fwd")
    st = lib.fa_fwd_shard(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), int(key_offset),
                          int(Nk_total), B, H, Nq, Nk, d, _scale(softmax_scale), ws.data_ptr(), ws.numel(),
                          _stream_ptr(q.device))
    _raise("fa_fwd_shard", st)
    return out, lse


def fa_bwd_shard(q, k, v, o, dout, lse, key_offset: int, Nk_total: int, softmax_scale=None, dq=None, dk=None,
                 dv=None, ws=None):
    """Backward of one causal key shard with the merged o and lse of all shards.
    Returns (partial dq, dk, dv of the shard) in bf16."""
    lib = load()
    B, Nq, H, d = q.shape
    Nk = k.shape[1]
    for name, t, shp in (("q", q, None), ("k", k, (B, Nk, H, d)), ("v", v, (B, Nk, H, d)), ("o", o, q.shape),
                         ("dout", dout, q.shape)):
        _check_tensor(name, t, torch.bfloat16, shp)
    _check_tensor("lse", lse, torch.float32, (B, H, Nq))
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if ws is None:
        ws = workspace(lib.fa_bwd_workspace_size(B, H, Nq, Nk, d), q.device, "bwd")
    st = lib.fa_bwd_shard(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dout.data_ptr(), lse.data_ptr(),
                          dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), int(key_offset), int(Nk_total), B, H, Nq, Nk,
                          d, _scale(softmax_scale), ws.data_ptr(), ws.numel(), _stream_ptr(q.device))
    _raise("fa_bwd_shard", st)
    return dq, dk, dv


def fa_merge_partials(o_parts, lse_parts, out=None, lse=None):
    """Merge shard results: o_parts [S, B, Nq, H, d] bf16, lse_parts [S, B, H, Nq] fp32
    -> (o [B, Nq, H, d], lse [B, H, Nq])."""
    lib = load()
    S, B, Nq, H, d = o_parts.shape
    _check_tensor("o_parts", o_parts, torch.bfloat16)
    _check_tensor("lse_parts", lse_parts, torch.float32, (S, B, H, Nq))
    out = torch.empty(o_parts.shape[1:], dtype=torch.bfloat16, device=o_parts.device) if out is None else out
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=o_parts.device) if lse is None else lse
    _check_tensor("out", out, torch.bfloat16, (B, Nq, H, d))
    _check_tensor("lse", lse, torch.float32, (B, H, Nq))
    st = lib.fa_merge_partials(o_parts.data_ptr(), lse_parts.data_ptr(), S, B, H, Nq, d, out.data_ptr(),
                               lse.data_ptr(), _stream_ptr(o_parts.device))
    _raise("fa_merge_partials", st)
    return out, lse


def fa_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, max_seqlen_k: int, causal: bool = False,
                  softmax_scale=None, out=None, lse=None, ws=None):
    """Forward over packed variable-length sequences.  q [total_q, H, d], k/v
    [total_k, H, d] bf16; cu_seqlens_q/k int32 [B+1] on the device.
    Returns (o [total_q, H, d] bf16, lse [H, total_q] fp32)."""
    lib = load()
    total_q, H, d = q.shape
    total_k = k.shape[0]
    B = cu_seqlens_q.shape[0] - 1
    _check_tensor("q", q, torch.bfloat16)
    _check_tensor("k", k, torch.bfloat16)
    _check_tensor("v", v, torch.bfloat16, k.shape)
    _check_tensor("cu_seqlens_q", cu_seqlens_q, torch.int32, (B + 1,))
    _check_tensor("cu_seqlens_k", cu_seqlens_k, torch.int32, (B + 1,))
    if k.dim() != 3 or k.shape[1] != H or k.shape[2] != d:
        raise ValueError("k/v must be [total_k, H, d]")
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((H, total_q), dtype=torch.float32, device=q.device) if lse is None else lse
    _check_tensor("out", out, torch.bfloat16, q.shape)
    _check_tensor("lse", lse, torch.float32, (H, total_q))
    if ws is None:
        ws = workspace(lib.fa_fwd_workspace_size(1, H, 1, 1, d), q.device, "fwd")
    st = lib.fa_fwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), cu_seqlens_q.data_ptr(),
                           cu_seqlens_k.data_ptr(), out.data_ptr(), lse.data_ptr(), B, H, total_q, total_k,
                           int(max_seqlen_q), int(max_seqlen_k), d, int(bool(causal)), _scale(softmax_scale),
                           ws.data_ptr(), ws.numel(), _stream_ptr(q.device))
    _raise("fa_fwd_varlen", st)
    return out, lse


def fa_bwd(q, k, v, o, dout, lse, causal: bool = False, softmax_scale=None, dq=None, dk=None, dv=None, ws=None):
    """Backward pass.  Returns (dq, dk, dv) in bf16, gradients of sum(O * dout)."""
    lib = load()
    B, Nq, H, d = q.shape
    Nk = k.shape[1]
    for name, t, shp in (("q", q, None), ("k", k, (B, Nk, H, d)), ("v", v, (B, Nk, H, d)), ("o", o, q.shape),
                         ("dout", dout, q.shape)):
        _check_tensor(name, t, torch.bfloat16, shp)
    _check_tensor("lse", lse, torch.float32, (B, H, Nq))
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = lib.fa_bwd_workspace_size(B, H, Nq, Nk, d)
    if ws is None:
        ws = workspace(need, q.device, "bwd")
    st = lib.fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dout.data_ptr(), lse.data_ptr(),
                    dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, Nq, Nk, d, int(bool(causal)),
                    _scale(softmax_scale), ws.data_ptr(), ws.numel(), _stream_ptr(q.device))
    _raise("fa_bwd", st)
    return dq, dk, dv


def fa_bwd_varlen(q, k, v, o, dout, lse, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, max_seqlen_k: int,
                  causal: bool = False, softmax_scale=None, dq=None, dk=None, dv=None, ws=None):
    """Backward over packed variable-length sequences (the inputs and lse of
    fa_fwd_varlen).  Returns (dq [total_q, H, d], dk, dv [total_k, H, d]) in bf16."""
    lib = load()
    total_q, H, d = q.shape
    total_k = k.shape[0]
    B = cu_seqlens_q.shape[0] - 1
    kshape = (total_k, H, d)
    for name, t, shp in (("q", q, None), ("k", k, kshape), ("v", v, kshape), ("o", o, q.shape),
                         ("dout", dout, q.shape)):
        _check_tensor(name, t, torch.bfloat16, shp)
    _check_tensor("lse", lse, torch.float32, (H, total_q))
    _check_tensor("cu_seqlens_q", cu_seqlens_q, torch.int32, (B + 1,))
    _check_tensor("cu_seqlens_k", cu_seqlens_k, torch.int32, (B + 1,))
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for name, t, shp in (("dq", dq, q.shape), ("dk", dk, kshape), ("dv", dv, kshape)):
        _check_tensor(name, t, torch.bfloat16, shp)
    if ws is None:
        ws = workspace(lib.fa_bwd_varlen_workspace_size(H, total_q, d), q.device, "bwd")
    st = lib.fa_bwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dout.data_ptr(), lse.data_ptr(),
                           dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), cu_seqlens_q.data_ptr(),
                           cu_seqlens_k.data_ptr(), B, H, total_q, total_k, int(max_seqlen_q), int(max_seqlen_k), d,
                           int(bool(causal)), _scale(softmax_scale), ws.data_ptr(), ws.numel(),
                           _stream_ptr(q.device))
    _raise("fa_bwd_varlen", st)
    return dq, dk, dv


def fa_decode_splitkv(q, k, v, cu_seqlens_k, max_seqlen_k: int, causal: bool = False, softmax_scale=None,
                      num_splits: int = 0, out=None, lse=None, ws=None):
    """Split-KV decode.  q [B, H, d]; k/v [total, H, d] bf16; cu_seqlens_k int32 [B+1] on the device.
    Returns (o [B, H, d] bf16, lse [B, H] fp32)."""
    lib = load()
    B, H, d = q.shape
    _check_tensor("q", q, torch.bfloat16)
    _check_tensor("k", k, torch.bfloat16)
    _check_tensor("v", v, torch.bfloat16, k.shape)
    _check_tensor("cu_seqlens_k", cu_seqlens_k, torch.int32, (B + 1,))
    if k.dim() != 3 or k.shape[1] != H or k.shape[2] != d:
        raise ValueError("k/v must be [total, H, d]")
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, H), dtype=torch.float32, device=q.device) if lse is None else lse
    need = lib.fa_decode_workspace_size(B, H, int(max_seqlen_k), d, int(num_splits))
    if ws is None:
        ws = workspace(need, q.device, "decode")
    st = lib.fa_decode_splitkv(q.data_ptr(), k.data_ptr(), v.data_ptr(), cu_seqlens_k.data_ptr(), B, H, 1,
                               int(max_seqlen_k), d, int(bool(causal)), _scale(softmax_scale), int(num_splits),
                               out.data_ptr(), lse.data_ptr(), ws.data_ptr(), ws.numel(), _stream_ptr(q.device))
    _raise("fa_decode_splitkv", st)
    return out, lse


def fa_decode_splitkv_checked(q, k, v, cu_seqlens_k, max_seqlen_k: int, softmax_scale=None, num_splits: int = 0,
                              out=None, lse=None, ws=None):
    """fa_decode_splitkv with every sequence's offsets checked on the device against
    the rows of k and v (k.shape[0]); a sequence outside them is skipped (its o and
    lse are not written) and fa_check then reports FA_ERR_INVALID_ARG."""
    lib = load()
    B, H, d = q.shape
    _check_tensor("q", q, torch.bfloat16)
    _check_tensor("k", k, torch.bfloat16)
    _check_tensor("v", v, torch.bfloat16, k.shape)
    _check_tensor("cu_seqlens_k", cu_seqlens_k, torch.int32, (B + 1,))
    if k.dim() != 3 or k.shape[1] != H or k.shape[2] != d:
        raise ValueError("k/v must be [total, H, d]")
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, H), dtype=torch.float32, device=q.device) if lse is None else lse
    _check_tensor("out", out, torch.bfloat16, q.shape)
    _check_tensor("lse", lse, torch.float32, (B, H))
    need = lib.fa_decode_workspace_size(B, H, int(max_seqlen_k), d, int(num_splits))
    if ws is None:
        ws = workspace(need, q.device, "decode")
    st = lib.fa_decode_splitkv_checked(q.data_ptr(), k.data_ptr(), v.data_ptr(), cu_seqlens_k.data_ptr(), B, H, 1,
                                       int(k.shape[0]), int(max_seqlen_k), d, 0, _scale(softmax_scale),
                                       int(num_splits), out.data_ptr(), lse.data_ptr(), ws.data_ptr(), ws.numel(),
                                       _stream_ptr(q.device))
    _raise("fa_decode_splitkv_checked", st)
    return out, lse


def fa_decode_splitkv_noalloc(q, k, v, cu_seqlens_k, max_seqlen_k: int, causal: bool = False, softmax_scale=None,
                              num_splits: int = 0, out=None, lse=None):
    """fa_decode_splitkv without a workspace: the library's own fixed 16 MiB device
    scratch holds the chunk states, for callers that cannot allocate device memory.
    Only the outputs below are allocated here, by torch, when not given."""
    lib = load()
    B, H, d = q.shape
    _check_tensor("q", q, torch.bfloat16)
    _check_tensor("k", k, torch.bfloat16)
    _check_tensor("v", v, torch.bfloat16, k.shape)
    _check_tensor("cu_seqlens_k", cu_seqlens_k, torch.int32, (B + 1,))
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, H), dtype=torch.float32, device=q.device) if lse is None else lse
    st = lib.fa_decode_splitkv_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), cu_seqlens_k.data_ptr(), B, H, 1,
                                       int(max_seqlen_k), d, int(bool(causal)), _scale(softmax_scale),
                                       int(num_splits), out.data_ptr(), lse.data_ptr(), _stream_ptr(q.device))
    _raise("fa_decode_splitkv_noalloc", st)
    return out, lse


def fa_decode_paged(q, k_pages, v_pages, block_table, seqlens_k, max_seqlen_k: int, softmax_scale=None,
                    num_splits: int = 0, out=None, lse=None, ws=None):
    """Split-KV decode over a paged cache.  q [B, H, d]; k_pages/v_pages
    [num_pages, page_size, H, d] bf16; block_table int32 [B, max_pages_per_seq] and
    seqlens_k int32 [B] on the device.  Returns (o [B, H, d] bf16, lse [B, H] fp32)."""
    lib = load()
    B, H, d = q.shape
    _check_tensor("q", q, torch.bfloat16)
    _check_tensor("k_pages", k_pages, torch.bfloat16)
    _check_tensor("v_pages", v_pages, torch.bfloat16, k_pages.shape)
    if k_pages.dim() != 4 or k_pages.shape[2] != H or k_pages.shape[3] != d:
        raise ValueError("k_pages/v_pages must be [num_pages, page_size, H, d]")
    if block_table.dim() != 2 or block_table.shape[0] != B:
        raise ValueError("block_table must be [B, max_pages_per_seq]")
    _check_tensor("block_table", block_table, torch.int32, tuple(block_table.shape))
    _check_tensor("seqlens_k", seqlens_k, torch.int32, (B,))
    num_pages, page_size = int(k_pages.shape[0]), int(k_pages.shape[1])
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, H), dtype=torch.float32, device=q.device) if lse is None else lse
    need = lib.fa_decode_workspace_size(B, H, int(max_seqlen_k), d, int(num_splits))
    if ws is None:
        ws = workspace(need, q.device, "decode")
    st = lib.fa_decode_paged(q.data_ptr(), k_pages.data_ptr(), v_pages.data_ptr(), block_table.data_ptr(),
                             seqlens_k.data_ptr(), B, H, num_pages, page_size, int(block_table.shape[1]),
                             int(max_seqlen_k), d, _scale(softmax_scale), int(num_splits), out.data_ptr(),
                             lse.data_ptr(), ws.data_ptr(), ws.numel(), _stream_ptr(q.device))
    _raise("fa_decode_paged", st)
    return out, lse


def fa_selftest_wait_timeout(ws: torch.Tensor, timeout_us: int = 1000) -> None:
    """Run the bounded-wait failure path once (see include/fa.h); read the result with fa_check."""
    _raise("fa_selftest_wait_timeout",
           load().fa_selftest_wait_timeout(ws.data_ptr(), ws.numel(), int(timeout_us), _stream_ptr(ws.device)))


def fa_check(ws: torch.Tensor) -> int:
    """Synchronise the current stream and return the kernels' status (0 = FA_OK)."""
    return int(load().fa_check(ws.data_ptr(), _stream_ptr(ws.device)))
