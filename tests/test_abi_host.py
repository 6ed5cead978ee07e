"""Host-side checks of the C ABI (no GPU needed): symbols, size queries, argument
validation and status strings.  Every call here returns before any kernel launch."""
import ctypes
import os
import re

import pytest

import exact_io_aware_54_b200 as fa
from exact_io_aware_54_b200 import build as fa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    fa_build.build()
    return fa.load()


def _declared_symbols():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            text = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"FA_API\s+[\w\s\*]+?\b(fa_\w+)\s*\(", text)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = _declared_symbols()
    assert {"fa_fwd", "fa_bwd", "fa_decode_splitkv", "fa_check"} <= set(names)
    raw = ctypes.CDLL(fa.lib_path())
    for n in names:
        assert hasattr(raw, n), f"{n} declared in include/ but not exported"


def test_version_and_status_strings(lib):
    assert re.fullmatch(r"\d+\.\d+\.\d+", fa.fa_version())
    for code, name in fa.STATUS.items():
        assert lib.fa_status_string(code).decode() == name
    assert lib.fa_status_string(99).decode() == "FA_ERR_UNKNOWN"


def test_workspace_sizes(lib):
    assert fa.fa_fwd_workspace_size(1, 2, 256, 256, 64) >= 4
    assert fa.fa_fwd_workspace_size(1, 2, 256, 256, 96) == 0
    assert fa.fa_fwd_workspace_size(0, 2, 256, 256, 64) == 0
    B, H, N, d = 64, 16, 1024, 64
    need = fa.fa_bwd_workspace_size(B, H, N, N, d)
    assert need >= 4 * B * N * H * d + 4 * B * H * N  # fp32 dQ accumulator + D rows
    # O(N) extra memory: far below one N x N score matrix per head
    assert fa.fa_bwd_workspace_size(1, 16, 16384, 16384, 64) < 16384 * 16384 * 2
    assert fa.fa_decode_workspace_size(1, 32, 8192, 128, 0) > 0
    assert fa.fa_decode_workspace_size(1, 32, 8192, 128, -1) == 0


def test_decode_split_plan(lib):
    for B, H, L, d, s in ((1, 32, 8192, 128, 0), (64, 32, 16384, 128, 0), (3, 5, 100, 64, 7), (2, 8, 1, 64, 0)):
        n = fa.fa_decode_num_splits(B, H, L, d, s)
        assert 1 <= n <= max(1, L)
        if s:
            assert n <= s
    assert fa.fa_decode_num_splits(4, 8, 1000, 64, 3) == 3


P = 0x10000  # a 16-byte aligned fake device address; validation fails before any use
ST = {v: k for k, v in fa.STATUS.items()}


def _fwd(lib, q=P, k=P, v=P, o=P, lse=P, B=1, H=1, Nq=8, Nk=8, d=64, ws=P, wsb=1 << 20):
    return lib.fa_fwd(q, k, v, o, lse, B, H, Nq, Nk, d, 0, 0.0, ws, wsb, None)


def test_fwd_argument_validation(lib):
    assert _fwd(lib, q=None) == ST["FA_ERR_INVALID_ARG"]
    assert _fwd(lib, B=0) == ST["FA_ERR_INVALID_ARG"]
    assert _fwd(lib, Nk=-3) == ST["FA_ERR_INVALID_ARG"]
    assert _fwd(lib, d=96) == ST["FA_ERR_UNSUPPORTED"]
    assert _fwd(lib, k=P + 8) == ST["FA_ERR_ALIGNMENT"]
    assert _fwd(lib, ws=None) == ST["FA_ERR_WORKSPACE"]
    assert _fwd(lib, wsb=1) == ST["FA_ERR_WORKSPACE"]


def test_bwd_argument_validation(lib):
    def call(**kw):
        a = dict(q=P, k=P, v=P, o=P, do=P, lse=P, dq=P, dk=P, dv=P, B=1, H=1, Nq=8, Nk=8, d=64, ws=P, wsb=1 << 30)
        a.update(kw)
        return lib.fa_bwd(a["q"], a["k"], a["v"], a["o"], a["do"], a["lse"], a["dq"], a["dk"], a["dv"], a["B"],
                          a["H"], a["Nq"], a["Nk"], a["d"], 1, 0.0, a["ws"], a["wsb"], None)

    assert call(do=None) == ST["FA_ERR_INVALID_ARG"]
    assert call(d=32) == ST["FA_ERR_UNSUPPORTED"]
    assert call(dv=P + 4) == ST["FA_ERR_ALIGNMENT"]
    assert call(wsb=16) == ST["FA_ERR_WORKSPACE"]


def test_decode_argument_validation(lib):
    def call(**kw):
        a = dict(q=P, k=P, v=P, cu=P, B=2, H=4, Nq=1, L=64, d=128, s=0, o=P, lse=P, ws=P, wsb=1 << 30)
        a.update(kw)
        return lib.fa_decode_splitkv(a["q"], a["k"], a["v"], a["cu"], a["B"], a["H"], a["Nq"], a["L"], a["d"], 0,
                                     0.0, a["s"], a["o"], a["lse"], a["ws"], a["wsb"], None)

    assert call(Nq=2) == ST["FA_ERR_INVALID_ARG"]
    assert call(cu=None) == ST["FA_ERR_INVALID_ARG"]
    assert call(s=-1) == ST["FA_ERR_INVALID_ARG"]
    assert call(d=80) == ST["FA_ERR_UNSUPPORTED"]
    assert call(o=P + 2) == ST["FA_ERR_ALIGNMENT"]
    assert call(cu=P + 2) == ST["FA_ERR_ALIGNMENT"]
    assert call(wsb=8) == ST["FA_ERR_WORKSPACE"]


def test_decode_checked_argument_validation(lib):
    def call(**kw):
        a = dict(q=P, k=P, v=P, cu=P, B=2, H=4, Nq=1, T=128, L=64, d=128, s=0, o=P, lse=P, ws=P, wsb=1 << 30)
        a.update(kw)
        return lib.fa_decode_splitkv_checked(a["q"], a["k"], a["v"], a["cu"], a["B"], a["H"], a["Nq"], a["T"],
                                             a["L"], a["d"], 0, 0.0, a["s"], a["o"], a["lse"], a["ws"], a["wsb"],
                                             None)

    assert call(T=-1) == ST["FA_ERR_INVALID_ARG"]
    assert call(Nq=2) == ST["FA_ERR_INVALID_ARG"]
    assert call(cu=None) == ST["FA_ERR_INVALID_ARG"]
    assert call(d=80) == ST["FA_ERR_UNSUPPORTED"]
    assert call(v=P + 2) == ST["FA_ERR_ALIGNMENT"]
    assert call(wsb=8) == ST["FA_ERR_WORKSPACE"]


def test_decode_paged_argument_validation(lib):
    def call(**kw):
        a = dict(q=P, k=P, v=P, bt=P, sl=P, B=2, H=4, npg=10, ps=16, mp=4, L=64, d=128, s=0, o=P, lse=P, ws=P,
                 wsb=1 << 30)
        a.update(kw)
        return lib.fa_decode_paged(a["q"], a["k"], a["v"], a["bt"], a["sl"], a["B"], a["H"], a["npg"], a["ps"],
                                   a["mp"], a["L"], a["d"], 0.0, a["s"], a["o"], a["lse"], a["ws"], a["wsb"], None)

    assert call(bt=None) == ST["FA_ERR_INVALID_ARG"]
    assert call(sl=None) == ST["FA_ERR_INVALID_ARG"]
    assert call(npg=0) == ST["FA_ERR_INVALID_ARG"]
    assert call(ps=0) == ST["FA_ERR_INVALID_ARG"]
    assert call(mp=0) == ST["FA_ERR_INVALID_ARG"]
    # 4 pages of 16 keys cannot hold a 65-key sequence
    assert call(L=65) == ST["FA_ERR_INVALID_ARG"]
    assert call(d=96) == ST["FA_ERR_UNSUPPORTED"]
    assert call(k=P + 8) == ST["FA_ERR_ALIGNMENT"]
    assert call(bt=P + 2) == ST["FA_ERR_ALIGNMENT"]
    assert call(sl=P + 1) == ST["FA_ERR_ALIGNMENT"]
    assert call(wsb=8) == ST["FA_ERR_WORKSPACE"]


def test_fwd_varlen_argument_validation(lib):
    def call(**kw):
        a = dict(q=P, k=P, v=P, cq=P, ck=P, o=P, lse=P, B=3, H=4, tq=300, tk=400, mq=200, mk=300, d=64, ws=P,
                 wsb=1 << 20)
        a.update(kw)
        return lib.fa_fwd_varlen(a["q"], a["k"], a["v"], a["cq"], a["ck"], a["o"], a["lse"], a["B"], a["H"],
                                 a["tq"], a["tk"], a["mq"], a["mk"], a["d"], 1, 0.0, a["ws"], a["wsb"], None)

    assert call(cq=None) == ST["FA_ERR_INVALID_ARG"]
    assert call(tk=0) == ST["FA_ERR_INVALID_ARG"]
    assert call(mq=0) == ST["FA_ERR_INVALID_ARG"]
    assert call(B=0) == ST["FA_ERR_INVALID_ARG"]
    assert call(d=80) == ST["FA_ERR_UNSUPPORTED"]
    assert call(o=P + 4) == ST["FA_ERR_ALIGNMENT"]
    assert call(ck=P + 2) == ST["FA_ERR_ALIGNMENT"]
    assert call(ws=None) == ST["FA_ERR_WORKSPACE"]


def test_bwd_varlen_argument_validation(lib):
    def call(**kw):
        a = dict(q=P, k=P, v=P, o=P, do=P, lse=P, dq=P, dk=P, dv=P, cq=P, ck=P, B=3, H=4, tq=300, tk=400, mq=200,
                 mk=300, d=64, ws=P, wsb=1 << 30)
        a.update(kw)
        return lib.fa_bwd_varlen(a["q"], a["k"], a["v"], a["o"], a["do"], a["lse"], a["dq"], a["dk"], a["dv"],
                                 a["cq"], a["ck"], a["B"], a["H"], a["tq"], a["tk"], a["mq"], a["mk"], a["d"], 1,
                                 0.0, a["ws"], a["wsb"], None)

    assert call(ck=None) == ST["FA_ERR_INVALID_ARG"]
    assert call(dk=None) == ST["FA_ERR_INVALID_ARG"]
    assert call(tq=0) == ST["FA_ERR_INVALID_ARG"]
    assert call(mk=0) == ST["FA_ERR_INVALID_ARG"]
    assert call(B=0) == ST["FA_ERR_INVALID_ARG"]
    assert call(tq=(1 << 31) - 100, H=1) == ST["FA_ERR_INVALID_ARG"]
    assert call(d=96) == ST["FA_ERR_UNSUPPORTED"]
    assert call(dv=P + 8) == ST["FA_ERR_ALIGNMENT"]
    assert call(cq=P + 2) == ST["FA_ERR_ALIGNMENT"]
    assert call(ws=None) == ST["FA_ERR_WORKSPACE"]
    need = fa.fa_bwd_varlen_workspace_size(4, 300, 64)
    assert need >= 4 * 300 * 4 * 64 + 4 * 4 * 300  # fp32 dQ accumulator + D rows
    assert call(wsb=need - 1) == ST["FA_ERR_WORKSPACE"]
    assert fa.fa_bwd_varlen_workspace_size(4, 300, 80) == 0


def test_masked_argument_validation(lib):
    def fwd(**kw):
        a = dict(q=P, k=P, v=P, o=P, lse=P, km=P, p=0.1, B=2, H=4, Nq=64, Nk=70, d=64, ws=P, wsb=1 << 20)
        a.update(kw)
        return lib.fa_fwd_masked(a["q"], a["k"], a["v"], a["o"], a["lse"], a["km"], a["p"], 7, a["B"], a["H"],
                                 a["Nq"], a["Nk"], a["d"], 1, 0.0, a["ws"], a["wsb"], None)

    def bwd(**kw):
        a = dict(q=P, k=P, v=P, o=P, do=P, lse=P, dq=P, dk=P, dv=P, km=P, p=0.0, B=2, H=4, Nq=64, Nk=70, d=128, ws=P,
                 wsb=1 << 30)
        a.update(kw)
        return lib.fa_bwd_masked(a["q"], a["k"], a["v"], a["o"], a["do"], a["lse"], a["dq"], a["dk"], a["dv"],
                                 a["km"], a["p"], 7, a["B"], a["H"], a["Nq"], a["Nk"], a["d"], 0, 0.0, a["ws"],
                                 a["wsb"], None)

    assert fwd(q=None) == ST["FA_ERR_INVALID_ARG"]
    assert fwd(Nk=0) == ST["FA_ERR_INVALID_ARG"]
    assert fwd(d=96) == ST["FA_ERR_UNSUPPORTED"]
    assert fwd(km=P + 2) == ST["FA_ERR_ALIGNMENT"]
    assert fwd(ws=None) == ST["FA_ERR_WORKSPACE"]
    assert fwd(p=-0.1) == ST["FA_ERR_INVALID_ARG"]
    assert fwd(p=1.0) == ST["FA_ERR_INVALID_ARG"]
    assert fwd(p=0.999995) == ST["FA_ERR_INVALID_ARG"]  # rounds to t = 65536: nothing would be kept
    assert fwd(p=float("nan")) == ST["FA_ERR_INVALID_ARG"]
    assert bwd(p=1.5) == ST["FA_ERR_INVALID_ARG"]
    assert bwd(dk=None) == ST["FA_ERR_INVALID_ARG"]
    assert bwd(km=P + 1) == ST["FA_ERR_ALIGNMENT"]


def test_blocksparse_argument_validation(lib):
    def fwd(**kw):
        a = dict(q=P, k=P, v=P, o=P, lse=P, bm=P, B=2, H=4, Nq=300, Nk=520, d=64, ws=P, wsb=1 << 20)
        a.update(kw)
        return lib.fa_fwd_blocksparse(a["q"], a["k"], a["v"], a["o"], a["lse"], a["bm"], a["B"], a["H"], a["Nq"],
                                      a["Nk"], a["d"], 1, 0.0, a["ws"], a["wsb"], None)

    def bwd(**kw):
        a = dict(q=P, k=P, v=P, o=P, do=P, lse=P, dq=P, dk=P, dv=P, bm=P, B=2, H=4, Nq=300, Nk=520, d=128, ws=P,
                 wsb=1 << 30)
        a.update(kw)
        return lib.fa_bwd_blocksparse(a["q"], a["k"], a["v"], a["o"], a["do"], a["lse"], a["dq"], a["dk"], a["dv"],
                                      a["bm"], a["B"], a["H"], a["Nq"], a["Nk"], a["d"], 0, 0.0, a["ws"], a["wsb"],
                                      None)

    assert fwd(bm=None) == ST["FA_ERR_INVALID_ARG"]
    assert fwd(q=None) == ST["FA_ERR_INVALID_ARG"]
    assert fwd(d=96) == ST["FA_ERR_UNSUPPORTED"]
    assert fwd(o=P + 4) == ST["FA_ERR_ALIGNMENT"]
    assert fwd(ws=None) == ST["FA_ERR_WORKSPACE"]
    assert bwd(bm=None) == ST["FA_ERR_INVALID_ARG"]
    assert bwd(dq=P + 8) == ST["FA_ERR_ALIGNMENT"]
    assert bwd(wsb=16) == ST["FA_ERR_WORKSPACE"]


def test_merge_partials_argument_validation(lib):
    def call(**kw):
        a = dict(op=P, lp=P, S=4, B=2, H=3, Nq=300, d=128, o=P, lse=P)
        a.update(kw)
        return lib.fa_merge_partials(a["op"], a["lp"], a["S"], a["B"], a["H"], a["Nq"], a["d"], a["o"], a["lse"],
                                     None)

    assert call(op=None) == ST["FA_ERR_INVALID_ARG"]
    assert call(S=0) == ST["FA_ERR_INVALID_ARG"]
    assert call(Nq=0) == ST["FA_ERR_INVALID_ARG"]
    assert call(d=96) == ST["FA_ERR_UNSUPPORTED"]
    assert call(o=P + 4) == ST["FA_ERR_ALIGNMENT"]
    assert call(lp=P + 8) == ST["FA_ERR_ALIGNMENT"]


def test_shard_argument_validation(lib):
    def fwd(**kw):
        a = dict(off=0, tot=1024, B=2, H=4, Nq=512, Nk=256, d=64)
        a.update(kw)
        return lib.fa_fwd_shard(P, P, P, P, P, a["off"], a["tot"], a["B"], a["H"], a["Nq"], a["Nk"], a["d"], 0.0,
                                P, 1 << 20, None)

    def bwd(**kw):
        a = dict(off=0, tot=1024, B=2, H=4, Nq=512, Nk=256, d=128)
        a.update(kw)
        return lib.fa_bwd_shard(P, P, P, P, P, P, P, P, P, a["off"], a["tot"], a["B"], a["H"], a["Nq"], a["Nk"],
                                a["d"], 0.0, P, 1 << 30, None)

    assert fwd(off=-1) == ST["FA_ERR_INVALID_ARG"]
    assert fwd(off=800) == ST["FA_ERR_INVALID_ARG"]   # 800 + 256 > 1024
    assert fwd(tot=0) == ST["FA_ERR_INVALID_ARG"]
    assert bwd(off=900) == ST["FA_ERR_INVALID_ARG"]
    assert bwd(Nk=2000) == ST["FA_ERR_INVALID_ARG"]


def test_selftest_argument_validation(lib):
    lib.fa_selftest_wait_timeout.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_uint, ctypes.c_void_p]
    assert lib.fa_selftest_wait_timeout(None, 256, 100, None) == ST["FA_ERR_WORKSPACE"]
    assert lib.fa_selftest_wait_timeout(P, 8, 100, None) == ST["FA_ERR_WORKSPACE"]
    assert lib.fa_selftest_wait_timeout(P + 4, 256, 100, None) == ST["FA_ERR_WORKSPACE"]
    assert lib.fa_selftest_wait_timeout(P, 256, 0, None) == ST["FA_ERR_INVALID_ARG"]
    assert lib.fa_selftest_wait_timeout(P, 256, 2000000, None) == ST["FA_ERR_INVALID_ARG"]


def test_check_rejects_null_workspace(lib):
    assert lib.fa_check(None, None) == ST["FA_ERR_INVALID_ARG"]


def test_binding_has_no_cpu_fallback(monkeypatch):
    """With the library missing, the binding raises instead of computing anything."""
    monkeypatch.setattr(fa, "_lib", None)
    monkeypatch.setenv("FA_LIB", "/nonexistent/libfa.so")
    with pytest.raises(ImportError):
        fa.load()
