"""The C-ABI library loads, exports every function include/*.h declares, and
rejects bad arguments on the host before launching anything (no GPU needed:
every call below returns before its first CUDA call)."""
import ctypes
import glob
import os
import re

import pytest

import sparse_attention_long_head_b200 as vs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"\b(vs_\w+)\s*\(", src):
            names.add(m.group(1))
    return names


def test_library_exports_every_declared_function():
    declared = _declared_functions()
    assert {"vs_select", "vs_sparse_attn_fwd", "vs_index_scores", "vs_dense_attn_fwd"} <= declared
    lib = vs.lib()
    for name in declared:
        assert hasattr(lib, name), name
        assert isinstance(getattr(lib, name), ctypes._CFuncPtr)
    assert set(vs.EXPORTS) == declared


def test_status_strings_and_version():
    assert vs.status_string(0) == "VS_OK"
    assert vs.status_string(5) == "VS_ERR_DEVICE_TIMEOUT"
    assert vs.status_string(99) == "VS_ERR_UNKNOWN"
    assert vs.vs_version() >= 100


def test_workspace_sizes():
    assert vs.vs_select_workspace_size(32, 131072) >= 256
    small = vs.vs_attn_workspace_size(1024, 1, 1, 64)
    big = vs.vs_attn_workspace_size(262144, 32, 8, 128)
    assert 256 < small < big
    # plan data is O(N) per index-set head: bitmaps + lists, no N x N structure
    assert big < 8 * 262144 * 4 * 4
    # room to pack the selected vertical K/V rows: 2 x H_sel x roundup(v_ld, 128) x d x 2 bytes
    packed = vs.vs_attn_workspace_size_ld(262144, 32, 8, 128, 16384)
    assert packed >= big + 2 * 8 * 16384 * 128 * 2
    assert vs.vs_attn_workspace_size_ld(1024, 1, 1, 64, 5) >= small + 2 * 128 * 64 * 2


P = ctypes.c_void_p


def _fake(addr=0x10000):
    return ctypes.c_void_p(addr)


def test_select_host_validation():
    L = vs.lib()
    ws = _fake(0x20000)
    good = dict(scores=_fake(), H=2, N=100, ld=100, mode=0, k=10, tau=0.5, idx=_fake(), ld_idx=10,
                cnt=_fake(), ws=ws, wsb=256)

    def call(**kw):
        a = dict(good)
        a.update(kw)
        return L.vs_select(a["scores"], a["H"], a["N"], a["ld"], a["mode"], a["k"], a["tau"],
                           a["idx"], a["ld_idx"], a["cnt"], a["ws"], a["wsb"], None)

    assert call(scores=None) == vs.VS_ERR_INVALID_ARG
    assert call(idx=None) == vs.VS_ERR_INVALID_ARG
    assert call(N=0) == vs.VS_ERR_INVALID_ARG
    assert call(ld=50) == vs.VS_ERR_INVALID_ARG
    assert call(k=0) == vs.VS_ERR_INVALID_ARG
    assert call(k=101) == vs.VS_ERR_INVALID_ARG
    assert call(ld_idx=5) == vs.VS_ERR_INVALID_ARG
    assert call(mode=7) == vs.VS_ERR_INVALID_ARG
    assert call(mode=1, tau=0.0) == vs.VS_ERR_INVALID_ARG
    assert call(mode=1, tau=1.5) == vs.VS_ERR_INVALID_ARG
    assert call(mode=1, tau=float("nan")) == vs.VS_ERR_INVALID_ARG
    assert call(mode=2, tau=0.0) == vs.VS_ERR_INVALID_ARG
    assert call(mode=2, tau=1.0000001) == vs.VS_ERR_INVALID_ARG
    assert call(mode=2, tau=float("nan")) == vs.VS_ERR_INVALID_ARG
    assert call(mode=3) == vs.VS_ERR_INVALID_ARG
    assert call(ws=None) == vs.VS_ERR_WORKSPACE
    assert call(wsb=16) == vs.VS_ERR_WORKSPACE
    assert call(ws=_fake(0x20010)) == vs.VS_ERR_WORKSPACE  # misaligned
    assert call(N=1 << 21, ld=1 << 21) == vs.VS_ERR_UNSUPPORTED


def test_select_varlen_host_validation():
    L = vs.lib()
    ws = _fake(0x20000)
    good = dict(scores=_fake(), total=1000, B=3, cu=_fake(0x30000), maxn=600, H=2, mode=1,
                caps=_fake(0x40000), cap_max=64, tau=0.9, idx=_fake(), ld_idx=64, cnt=_fake(),
                ws=ws, wsb=256)

    def call(**kw):
        a = dict(good)
        a.update(kw)
        return L.vs_select_varlen(a["scores"], a["total"], a["B"], a["cu"], a["maxn"], a["H"],
                                  a["mode"], a["caps"], a["cap_max"], a["tau"], a["idx"],
                                  a["ld_idx"], a["cnt"], a["ws"], a["wsb"], None)

    assert vs.vs_select_workspace_size_varlen(3, 2, 600) >= 256
    for bad in ("scores", "cu", "caps", "idx", "cnt"):
        assert call(**{bad: None}) == vs.VS_ERR_INVALID_ARG, bad
    assert call(B=0) == vs.VS_ERR_INVALID_ARG
    assert call(H=0) == vs.VS_ERR_INVALID_ARG
    assert call(B=40000, H=2) == vs.VS_ERR_INVALID_ARG  # more than 65535 rows
    assert call(maxn=0) == vs.VS_ERR_INVALID_ARG
    assert call(total=0) == vs.VS_ERR_INVALID_ARG
    assert call(cap_max=0) == vs.VS_ERR_INVALID_ARG
    assert call(ld_idx=63) == vs.VS_ERR_INVALID_ARG
    assert call(mode=7) == vs.VS_ERR_INVALID_ARG
    assert call(tau=0.0) == vs.VS_ERR_INVALID_ARG
    assert call(mode=2, tau=1.5) == vs.VS_ERR_INVALID_ARG
    assert call(ws=None) == vs.VS_ERR_WORKSPACE
    assert call(wsb=16) == vs.VS_ERR_WORKSPACE
    assert call(ws=_fake(0x20010)) == vs.VS_ERR_WORKSPACE
    assert call(maxn=(1 << 20) + 1) == vs.VS_ERR_UNSUPPORTED


def test_attention_host_validation():
    L = vs.lib()
    f = _fake
    base = dict(Q=f(0x1000), K=f(0x2000), V=f(0x3000), dtype=0, N=256, Hq=4, Hkv=2, d=128,
                qs=512, kvs=256, scale=0.0, Hsel=4, vi=f(0x4000), vld=8, vc=f(0x5000),
                si=f(0x6000), sld=8, sc=f(0x7000), O=f(0x8000), lse=None, ws=f(0x10000),
                wsb=1 << 30)

    def call(**kw):
        a = dict(base)
        a.update(kw)
        return L.vs_sparse_attn_fwd(a["Q"], a["K"], a["V"], a["dtype"], a["N"], a["Hq"], a["Hkv"],
                                    a["d"], a["qs"], a["kvs"], a["scale"], a["Hsel"], a["vi"],
                                    a["vld"], a["vc"], a["si"], a["sld"], a["sc"], a["O"],
                                    a["lse"], a["ws"], a["wsb"], None)

    assert call(Q=None) == vs.VS_ERR_INVALID_ARG
    assert call(O=None) == vs.VS_ERR_INVALID_ARG
    assert call(vi=None) == vs.VS_ERR_INVALID_ARG
    assert call(Hkv=3) == vs.VS_ERR_INVALID_ARG
    assert call(Hsel=3) == vs.VS_ERR_INVALID_ARG
    assert call(d=96, qs=384, kvs=192) == vs.VS_ERR_UNSUPPORTED
    assert call(qs=100) == vs.VS_ERR_INVALID_ARG
    assert call(qs=516, kvs=260) == vs.VS_ERR_UNSUPPORTED  # rows not 16-byte multiples
    assert call(scale=-1.0) == vs.VS_ERR_INVALID_ARG
    assert call(scale=float("inf")) == vs.VS_ERR_INVALID_ARG
    assert call(dtype=5) == vs.VS_ERR_INVALID_ARG
    assert call(Q=f(0x1008)) == vs.VS_ERR_UNSUPPORTED  # misaligned
    assert call(ws=None) == vs.VS_ERR_WORKSPACE
    assert call(wsb=1000) == vs.VS_ERR_WORKSPACE
    assert call(N=0) == vs.VS_ERR_INVALID_ARG
    rc = L.vs_dense_attn_fwd(None, f(), f(), 0, 10, 1, 1, 64, 64, 64, 0.0, f(), None, f(), 256, None)
    assert rc == vs.VS_ERR_INVALID_ARG


def test_varlen_host_validation():
    L = vs.lib()
    f = _fake
    base = dict(Q=f(0x1000), K=f(0x2000), V=f(0x3000), dtype=0, T=1000, B=3, cu=f(0x9000),
                maxn=500, Hq=4, Hkv=2, d=128, qs=512, kvs=256, scale=0.0, Hsel=2, vi=f(0x4000),
                vld=8, vc=f(0x5000), si=f(0x6000), sld=8, sc=f(0x7000), O=f(0x8000), lse=None,
                ws=f(0x10000), wsb=1 << 30)

    def call(**kw):
        a = dict(base)
        a.update(kw)
        return L.vs_sparse_attn_fwd_varlen(a["Q"], a["K"], a["V"], a["dtype"], a["T"], a["B"],
                                           a["cu"], a["maxn"], a["Hq"], a["Hkv"], a["d"], a["qs"],
                                           a["kvs"], a["scale"], a["Hsel"], a["vi"], a["vld"],
                                           a["vc"], a["si"], a["sld"], a["sc"], a["O"], a["lse"],
                                           a["ws"], a["wsb"], None)

    assert call(cu=None) == vs.VS_ERR_INVALID_ARG
    assert call(B=0) == vs.VS_ERR_INVALID_ARG
    assert call(T=0) == vs.VS_ERR_INVALID_ARG
    assert call(maxn=0) == vs.VS_ERR_INVALID_ARG
    assert call(dtype=1) == vs.VS_ERR_UNSUPPORTED
    assert call(Hsel=3) == vs.VS_ERR_INVALID_ARG
    assert call(wsb=1000) == vs.VS_ERR_WORKSPACE
    rc = L.vs_dense_attn_fwd_varlen(f(), f(), f(), 0, 100, 2, None, 50, 1, 1, 64, 64, 64, 0.0,
                                    f(), None, f(0x10000), 256, None)
    assert rc == vs.VS_ERR_INVALID_ARG
    # the plan grows with the batch; packing needs room for every slot
    one = vs.vs_attn_workspace_size_varlen(1, 4096, 4, 128, 0)
    assert one == vs.vs_attn_workspace_size(4096, 4, 4, 128)
    assert vs.vs_attn_workspace_size_varlen(3, 4096, 4, 128, 0) > 2 * one
    assert vs.vs_attn_workspace_size_varlen(3, 4096, 4, 128, 256) >= \
        vs.vs_attn_workspace_size_varlen(3, 4096, 4, 128, 0) + 2 * 12 * 256 * 128 * 2


def test_aggregate_host_validation():
    L = vs.lib()
    f = _fake
    base = dict(Q=f(0x1000), K=f(0x2000), dtype=0, N=256, Hq=4, Hkv=2, d=128, qs=512, kvs=256,
                scale=0.0, lse=f(0x3000), Av=f(0x4000), As=f(0x5000), ws=f(0x10000), wsb=256)

    def call(**kw):
        a = dict(base)
        a.update(kw)
        return L.vs_attn_aggregate(a["Q"], a["K"], a["dtype"], a["N"], a["Hq"], a["Hkv"], a["d"],
                                   a["qs"], a["kvs"], a["scale"], a["lse"], a["Av"], a["As"],
                                   a["ws"], a["wsb"], None)

    assert call(lse=None) == vs.VS_ERR_INVALID_ARG
    assert call(Av=None) == vs.VS_ERR_INVALID_ARG
    assert call(As=None) == vs.VS_ERR_INVALID_ARG
    assert call(Q=None) == vs.VS_ERR_INVALID_ARG
    assert call(Hkv=3) == vs.VS_ERR_INVALID_ARG
    assert call(d=96, qs=384, kvs=192) == vs.VS_ERR_UNSUPPORTED
    assert call(dtype=1) == vs.VS_ERR_UNSUPPORTED
    assert call(ws=None) == vs.VS_ERR_WORKSPACE
    assert call(wsb=100) == vs.VS_ERR_WORKSPACE
    assert call(N=0) == vs.VS_ERR_INVALID_ARG


def test_indexer_and_misc_host_validation():
    L = vs.lib()
    f = _fake
    assert L.vs_index_scores(None, f(), 0, 10, 2, 64, 128, 64, f(), f(), 256, f(), f(), None) == \
        vs.VS_ERR_INVALID_ARG
    assert L.vs_index_scores(f(), f(), 0, 10, 2, 64, 128, 64, f(), f(), 0, f(), f(), None) == \
        vs.VS_ERR_INVALID_ARG
    assert L.vs_index_scores(f(), f(), 0, 10, 2, 64, 100, 64, f(), f(), 256, f(), f(), None) == \
        vs.VS_ERR_INVALID_ARG
    flags = ctypes.c_int(0)
    assert L.vs_read_device_status(None, None, ctypes.byref(flags)) == vs.VS_ERR_INVALID_ARG
    assert L.vs_selftest_wait_timeout(None, 1000000, None) == vs.VS_ERR_WORKSPACE
    assert L.vs_selftest_wait_timeout(f(0x10000), 10, None) == vs.VS_ERR_INVALID_ARG
    assert L.vs_selftest_exp(None, f(0x10000), 4, None) == vs.VS_ERR_INVALID_ARG
    assert L.vs_selftest_exp(f(0x10000), f(0x20000), 0, None) == vs.VS_ERR_INVALID_ARG


def test_binding_has_no_cpu_fallback(monkeypatch, tmp_path):
    # a missing library must fail loudly, never silently compute elsewhere
    monkeypatch.setattr(vs, "_lib", None)
    monkeypatch.setattr(vs, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        vs.lib()
