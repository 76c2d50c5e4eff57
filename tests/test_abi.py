"""The C ABI on a machine without a GPU: the library loads, exports every
entry point include/qsa.h declares, and rejects bad arguments on the host
(before any CUDA call) with the documented status codes."""
import ctypes
import os
import re

import pytest

import block_sparse_long_10_b200 as qsa
from block_sparse_long_10_b200 import build as qbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
OK, INVALID, UNSUPPORTED, WORKSPACE = 0, 1, 2, 3
SIZE_MAX = ctypes.c_size_t(-1).value


@pytest.fixture(scope="module")
def lib():
    qbuild.build()
    return qsa.load()


def _declared():
    with open(os.path.join(ROOT, "include", "qsa.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"QSA_API\s+[\w\s\*]*?\b(qsa_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert len(names) >= 14, names
    for n in names:
        assert hasattr(lib, n), n


def test_no_internal_symbols_exported(lib):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", qsa.lib_path()],
                         capture_output=True, text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    ours = {s for s in exported if s.startswith("qsa_")}
    assert ours == set(_declared())
    assert not any("qsa3" in s for s in exported)  # no mangled qsa:: internals


def test_status_strings_and_version(lib):
    assert qsa.qsa_status_string(0) == "ok"
    assert "workspace" in qsa.qsa_status_string(3)
    assert qsa.qsa_version().count(".") == 2


def _nullp():
    return ctypes.c_void_p(0)


def _fake(n=0x10000):
    # a 16-byte aligned non-null address; never dereferenced by host validation
    return ctypes.c_void_p(n)


def test_pool_validation(lib):
    s = _nullp()
    assert lib.qsa_pool(_fake(), 1, 64, 64, 0, 0, 16, _fake(), s) == INVALID      # r <= 0
    assert lib.qsa_pool(_fake(), 1, 64, 64, 4, 0, 17, _fake(), s) == INVALID      # range
    assert lib.qsa_pool(_fake(), 1, 64, 64, 4, 5, 4, _fake(), s) == INVALID       # inverted
    assert lib.qsa_pool(_fake(), 1, 64, 64, 2, 0, 8, _fake(), s) == UNSUPPORTED   # r != 4
    assert lib.qsa_pool(_fake(), 1, 64, 60, 4, 0, 16, _fake(), s) == UNSUPPORTED  # Di % 8
    assert lib.qsa_pool(_nullp(), 1, 64, 64, 4, 0, 16, _fake(), s) == INVALID     # null
    assert lib.qsa_pool(_fake(), 1, 64, 64, 4, 3, 3, _fake(), s) == OK            # empty range
    assert lib.qsa_pool(_fake(8), 1, 64, 64, 4, 0, 16, _fake(), s) == INVALID     # misaligned


def test_index_topk_validation(lib):
    f, s = _fake(), _nullp()
    ws_n = lib.qsa_index_topk_workspace_size(1, 2048, 512, 4, 64, 4, 2048)
    assert 256 < ws_n < SIZE_MAX
    args = lambda **kw: dict(dict(q=f, w=f, kp=f, pos=None, B=1, Tq=2048, N=512, Hi=4, Di=64,
                                  r=4, budget=2048, sel=f, sc=None, ws=f, wsb=ws_n), **kw)
    call = lambda a: lib.qsa_index_topk(a["q"], a["w"], a["kp"], a["pos"], a["B"], a["Tq"],
                                        a["N"], a["Hi"], a["Di"], a["r"], a["budget"], a["sel"],
                                        a["sc"], a["ws"], a["wsb"], s)
    assert call(args(budget=2047)) == INVALID
    assert call(args(B=0)) == INVALID
    assert call(args(q=_nullp())) == INVALID
    assert call(args(kp=_nullp())) == INVALID           # pooled keys needed when N > 0
    assert call(args(N=100)) == INVALID                 # queries beyond the pooled keys
    assert call(args(Hi=3)) == UNSUPPORTED
    assert call(args(Di=48)) == UNSUPPORTED
    assert call(args(budget=4096)) == UNSUPPORTED       # kb - 1 > 511
    assert call(args(r=8, budget=2048, N=256)) == UNSUPPORTED
    assert call(args(wsb=ws_n - 1)) == WORKSPACE
    assert call(args(ws=_nullp())) == WORKSPACE
    assert call(args(Tq=0)) == OK
    assert lib.qsa_index_topk_workspace_size(0, 1, 1, 1, 32, 4, 8) == SIZE_MAX
    assert lib.qsa_index_topk_decode_workspace_size(64, 65536, 4, 2048) > 64 * 16 * 511 * 8
    assert lib.qsa_index_topk_decode_workspace_size(1, 1, 4, 6) == SIZE_MAX


def test_attention_validation(lib):
    f, s = _fake(), _nullp()
    sp = lambda **kw: lib.qsa_sparse_attn_prefill(
        f, f, f, f, None, kw.get("B", 1), kw.get("Tq", 64), kw.get("Tk", 64), kw.get("Hq", 16),
        kw.get("Hkv", 2), kw.get("D", 128), 4, kw.get("budget", 2048), ctypes.c_float(0.1),
        f, None, s)
    assert sp(Hq=15) == INVALID
    assert sp(D=96) == UNSUPPORTED
    assert sp(Hq=48, Hkv=2) == UNSUPPORTED             # G = 24
    assert sp(Tq=65) == INVALID                        # queries beyond K/V without q_pos0
    assert sp(budget=8192) == UNSUPPORTED               # kb > 1024
    assert sp(Tq=0) == OK
    assert sp(Tq=0, Tk=0) == OK                        # empty sequence: no-op
    assert sp(Tk=0) == INVALID
    nan = ctypes.c_float(float("nan"))
    assert lib.qsa_dense_gqa_prefill(f, f, f, 1, 64, 16, 2, 128, nan, f, None, s) == INVALID
    assert lib.qsa_dense_gqa_prefill(f, f, f, 1, 64, 16, 2, 80, ctypes.c_float(.1), f, None,
                                     s) == UNSUPPORTED
    n = lib.qsa_sparse_attn_decode_workspace_size(64, 16, 128, 4, 2048)
    assert lib.qsa_sparse_attn_decode(f, f, f, f, 4096, f, 64, 16, 2, 128, 4, 2048,
                                      ctypes.c_float(.1), f, None, f, n - 4, s) == WORKSPACE
    m = lib.qsa_dense_gqa_decode_workspace_size(64, 262144, 16, 128)
    assert m > 64 * 16 * 130 * 4
    assert lib.qsa_dense_gqa_decode(f, f, f, f, 262144, 64, 16, 2, 128, ctypes.c_float(.1),
                                    f, None, f, m - 1, s) == WORKSPACE


def test_index_distill_validation(lib):
    f, s = _fake(), _nullp()
    n = lib.qsa_index_distill_workspace_size(1, 2048, 1, 4)
    assert n == 256 + 2048 * 512 * 4 + 2048 * 8
    assert lib.qsa_index_distill_workspace_size(1, 2048, 1, 2) == SIZE_MAX
    assert lib.qsa_index_distill_workspace_size(0, 2048, 1, 4) == SIZE_MAX
    base = dict(q=f, k=f, lse=f, qi=f, w=f, kp=f, B=1, T=2048, Hq=4, Hkv=1, D=64, Hi=2, Di=32,
                r=4, scale=ctypes.c_float(0.125), kl=f, dq=f, dw=f, dkp=f, dki=None, ws=f, wsb=n)
    call = lambda **kw: lib.qsa_index_distill(*dict(base, **kw).values(), s)
    assert call(Hq=5, Hkv=2) == INVALID                  # Hq % Hkv
    assert call(lse=_nullp()) == INVALID
    assert call(dkp=_nullp()) == INVALID                 # needed when T >= r
    assert call(scale=ctypes.c_float(float("nan"))) == INVALID
    assert call(r=8) == UNSUPPORTED
    assert call(D=96) == UNSUPPORTED
    assert call(Hi=3) == UNSUPPORTED
    assert call(Hq=16, Hkv=1) == UNSUPPORTED             # G = 16
    assert call(wsb=n - 1) == WORKSPACE
    assert call(ws=_nullp()) == WORKSPACE
    assert call(q=_fake(0x10008)) == INVALID              # misaligned
    assert call(T=0) == OK


def test_sparse_attn_backward_validation(lib):
    f, s = _fake(), _nullp()
    base = dict(q=f, k=f, v=f, sel=f, do=f, B=1, T=64, Hq=16, Hkv=2, D=128, r=4, budget=2048,
                scale=ctypes.c_float(0.1), dq=f, dk=f, dv=f)
    call = lambda **kw: lib.qsa_sparse_attn_backward(*dict(base, **kw).values(), s)
    assert call(Hq=15) == INVALID
    assert call(budget=2047) == INVALID
    assert call(do=_nullp()) == INVALID
    assert call(dk=_fake(0x10004)) == INVALID               # misaligned
    assert call(D=96) == UNSUPPORTED
    assert call(r=2, budget=2048) == UNSUPPORTED
    assert call(budget=8192) == UNSUPPORTED                 # kb > 1024
    assert call(T=0) == OK


def test_gdn_validation(lib):
    f, s = _fake(), _nullp()
    pre = lambda **kw: lib.qsa_gdn_prefill(*dict(dict(
        q=f, k=f, v=f, a=f, b=f, s0=None, B=1, T=64, H=4, dk=128, dv=128, o=f, s1=f),
        **kw).values(), s)
    assert pre(H=0) == INVALID
    assert pre(s1=_nullp()) == INVALID
    assert pre(a=_nullp()) == INVALID
    assert pre(dk=96) == UNSUPPORTED
    assert pre(s1=_fake(0x10008)) == INVALID                 # misaligned state
    dec = lambda **kw: lib.qsa_gdn_decode(*dict(dict(
        q=f, k=f, v=f, a=f, b=f, st=f, B=2, H=4, dk=64, dv=64, o=f), **kw).values(), s)
    assert dec(B=0) == INVALID
    assert dec(st=_nullp()) == INVALID
    assert dec(dv=32) == UNSUPPORTED
    # the chunked prefill: its workspace size, then the same checks plus the workspace
    assert lib.qsa_gdn_prefill_chunked_workspace_size(1, 64, 4, 128, 128) == 256 + 4 * 115200
    assert lib.qsa_gdn_prefill_chunked_workspace_size(1, 65, 4, 64, 64) == 256 + 2 * 4 * 66048
    assert lib.qsa_gdn_prefill_chunked_workspace_size(1, 64, 4, 96, 128) == SIZE_MAX
    big = 1 << 24
    chk = lambda **kw: lib.qsa_gdn_prefill_chunked(*dict(dict(
        q=f, k=f, v=f, a=f, b=f, s0=None, B=1, T=64, H=4, dk=128, dv=128, o=f, s1=f, ws=f,
        n=big), **kw).values(), s)
    assert chk(H=0) == INVALID
    assert chk(dk=96) == UNSUPPORTED
    assert chk(ws=_nullp()) == WORKSPACE
    assert chk(n=1000) == WORKSPACE
    assert chk(ws=_fake(0x10010)) == WORKSPACE              # not 256-byte aligned


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(qsa, "_LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(qsa, "_lib", None)
    with pytest.raises(qsa.QSAError):
        qsa.load()
