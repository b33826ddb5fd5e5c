"""The C-ABI library loads, exports every symbol that include/csa2.h declares, and rejects
invalid arguments on the host (before any CUDA call, so these run without a GPU)."""
import ctypes
import os
import re

import pytest

import sparse_attention_decode_kv_b200 as csa2
from sparse_attention_decode_kv_b200 import build as csa2_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "csa2.h")

OK, INVALID, UNSUPPORTED, WORKSPACE = 0, -1, -2, -3
FAKE = 1 << 20          # an aligned, never-dereferenced address
MIS = (1 << 20) + 4     # misaligned


@pytest.fixture(scope="module")
def L():
    csa2_build.build()
    return csa2.lib()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"CSA2_API\s+[\w\s\*]+?\b(csa2_\w+)\s*\(", text)))


def test_header_declares_the_four_entry_points():
    names = declared_functions()
    for n in ("csa2_append_quant", "csa2_index_full", "csa2_index_reindex", "csa2_attend"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def test_status_strings_and_version(L):
    assert csa2.status_string(0) == "CSA2_OK"
    for s in (-1, -2, -3, -4, -5, -6):
        assert csa2.status_string(s).startswith("CSA2_ERR")
    assert L.csa2_abi_version() == 3
    assert csa2.launch_count() >= 0


def test_workspace_sizes(L):
    ws = csa2.index_full_workspace_bytes(8, 1 << 20, 512, 2048)
    # scores + block maxima + histograms + counters + candidates
    assert ws >= 8 * (1 << 20) * 4 + 8 * (1 << 17) * 4
    assert ws % 256 == 0
    assert csa2.index_full_workspace_bytes(0, 8, 1, 1) == 0
    assert csa2.index_reindex_workspace_bytes(8, 16384, 512) == 8 * 16384 * 8
    assert csa2.attend_workspace_bytes(8, 512, 128) > 0          # split over tiles
    assert csa2.attend_workspace_bytes(4096, 512, 128) == 0      # one CTA per sequence


def P(v):
    return ctypes.c_void_p(v) if v else None


def append(L, **kw):
    a = dict(x=FAKE, ik=FAKE, B=2, n=4, pos=FAKE, n_cap=64, codes=FAKE, scales=FAKE,
             ik_cache=FAKE, swa=FAKE, swa_scale=FAKE, W=8, dev_err=None)
    a.update(kw)
    return L.csa2_append_quant(P(a["x"]), P(a["ik"]), a["B"], a["n"], P(a["pos"]), a["n_cap"],
                               P(a["codes"]), P(a["scales"]), P(a["ik_cache"]), P(a["swa"]),
                               P(a["swa_scale"]), a["W"], P(a["dev_err"]), None)


def test_append_rejects_bad_arguments(L):
    assert append(L, B=0) == INVALID
    assert append(L, n=-1) == INVALID
    assert append(L, n_cap=60) == INVALID            # not a multiple of 8
    assert append(L, x=0) == INVALID
    assert append(L, codes=MIS) == INVALID
    assert append(L, ik=0) == INVALID                # ik and ik_cache must both be given or not
    assert append(L, swa=0) == INVALID               # ring needs both arrays
    assert append(L, swa=0, swa_scale=0) == INVALID  # W > 0 without a ring
    assert append(L, dev_err=FAKE + 2) == INVALID
    assert append(L, B=5000) == UNSUPPORTED
    assert append(L, W=5000) == UNSUPPORTED
    assert append(L, n=0) == OK                      # nothing to do: no launch


def ced(L, **kw):
    a = dict(h=FAKE, w=FAKE, B=2, n=100, d=256, pos=FAKE, n_cap=64, codes=FAKE, scales=FAKE,
             dev_err=None)
    a.update(kw)
    return L.csa2_ced_project_quant(P(a["h"]), P(a["w"]), a["B"], a["n"], a["d"], P(a["pos"]),
                                    a["n_cap"], P(a["codes"]), P(a["scales"]), P(a["dev_err"]),
                                    None)


def test_ced_projection_rejects_bad_arguments(L):
    assert ced(L, B=0) == INVALID
    assert ced(L, n=-1) == INVALID
    assert ced(L, d=0) == INVALID
    assert ced(L, d=100) == INVALID                  # not a multiple of 64
    assert ced(L, n_cap=60) == INVALID
    assert ced(L, h=0) == INVALID
    assert ced(L, w=MIS) == INVALID
    assert ced(L, scales=0) == INVALID
    assert ced(L, dev_err=FAKE + 2) == INVALID
    assert ced(L, d=65600) == UNSUPPORTED
    assert ced(L, B=4096, n=1 << 15) == UNSUPPORTED  # more than 2^26 tokens
    assert ced(L, n=0) == OK                         # nothing to do: no launch


def replay(L, ws_bytes=1 << 30, **kw):
    a = dict(h=FAKE, w=FAKE, B=2, Wr=128, d=256, N=FAKE, swa=FAKE, swa_scale=FAKE, W=128, ws=FAKE,
             dev_err=None)
    a.update(kw)
    return L.csa2_swa_replay(P(a["h"]), P(a["w"]), a["B"], a["Wr"], a["d"], P(a["N"]), P(a["swa"]),
                             P(a["swa_scale"]), a["W"], P(a["ws"]), ws_bytes, P(a["dev_err"]), None)


def test_swa_replay_rejects_bad_arguments(L):
    assert replay(L, B=0) == INVALID
    assert replay(L, Wr=-1) == INVALID
    assert replay(L, Wr=129) == INVALID              # more window rows than ring slots
    assert replay(L, W=0) == INVALID
    assert replay(L, d=96) == INVALID                # not a multiple of 64
    assert replay(L, h=0) == INVALID
    assert replay(L, w=MIS) == INVALID
    assert replay(L, N=0) == INVALID
    assert replay(L, swa_scale=0) == INVALID
    assert replay(L, dev_err=FAKE + 2) == INVALID
    assert replay(L, d=65600) == UNSUPPORTED
    assert replay(L, W=8192, Wr=8) == UNSUPPORTED
    assert replay(L, ws_bytes=16) == WORKSPACE
    assert replay(L, ws=0) == WORKSPACE
    assert replay(L, Wr=0) == OK                      # nothing to do: no launch


def test_swa_replay_workspace_size(L):
    # 2 x 128 rows = 2 token tiles x 2 channel halves = 4 tiles; the d-slices split 37 ways
    # (148 / 4) but never more than d / 64
    assert csa2.swa_replay_workspace_bytes(2, 128, 4096) == 37 * 256 * 512 * 4
    assert csa2.swa_replay_workspace_bytes(2, 128, 256) == 4 * 256 * 512 * 4
    assert csa2.swa_replay_workspace_bytes(8, 4096, 64) == 1 * 8 * 4096 * 512 * 4
    assert csa2.swa_replay_workspace_bytes(0, 128, 256) == 0
    assert csa2.swa_replay_workspace_bytes(2, 128, 100) == 0


def cache_copy(L, fn, N=(5, 7), **kw):
    a = dict(dc=FAKE, ds=FAKE, di=FAKE, B=2, n_cap=64, n_host=32, hc=FAKE, hs=FAKE, hi=FAKE)
    a.update(kw)
    n = (ctypes.c_int32 * len(N))(*N)
    if fn == "restore":
        return L.csa2_cache_restore(P(a["hc"]), P(a["hs"]), P(a["hi"]), a["B"], a["n_host"], n,
                                    a["n_cap"], P(a["dc"]), P(a["ds"]), P(a["di"]), None)
    return L.csa2_cache_persist(P(a["dc"]), P(a["ds"]), P(a["di"]), a["B"], a["n_cap"], n,
                                a["n_host"], P(a["hc"]), P(a["hs"]), P(a["hi"]), None)


@pytest.mark.parametrize("fn", ["restore", "persist"])
def test_cache_copies_reject_bad_arguments(L, fn):
    assert cache_copy(L, fn, B=0) == INVALID
    assert cache_copy(L, fn, n_cap=60) == INVALID    # not a multiple of 8
    assert cache_copy(L, fn, n_host=-1) == INVALID
    assert cache_copy(L, fn, N=(5, 33)) == INVALID   # more rows than the host layout holds
    assert cache_copy(L, fn, N=(5, 70), n_host=128) == INVALID  # more than the cache holds
    assert cache_copy(L, fn, N=(-1, 3)) == INVALID
    assert cache_copy(L, fn, dc=0) == INVALID
    assert cache_copy(L, fn, hs=MIS) == INVALID
    assert cache_copy(L, fn, hi=0) == INVALID        # keys on one side only
    assert cache_copy(L, fn, di=0, hi=0, B=5000, N=(0,) * 5000) == UNSUPPORTED


def index_full(L, ws_bytes=None, **kw):
    a = dict(iq=FAKE, w=FAKE, ik=FAKE, N=FAKE, B=2, n_cap=1024, K=64, P=32, topk=FAKE,
             pool=FAKE, ws=FAKE)
    a.update(kw)
    if ws_bytes is None:
        ws_bytes = 0
    return L.csa2_index_full(P(a["iq"]), P(a["w"]), P(a["ik"]), P(a["N"]), a["B"], a["n_cap"],
                             a["K"], a["P"], P(a["topk"]), P(a["pool"]), P(a["ws"]), ws_bytes,
                             None, None)


def test_index_full_rejects_bad_arguments(L):
    assert index_full(L, B=0) == INVALID
    assert index_full(L, K=0) == INVALID
    assert index_full(L, P=0) == INVALID
    assert index_full(L, n_cap=100) == INVALID
    assert index_full(L, iq=MIS) == INVALID
    assert index_full(L, ws=0) == INVALID
    assert index_full(L, K=5000) == UNSUPPORTED
    assert index_full(L, P=5000) == UNSUPPORTED
    need = csa2.index_full_workspace_bytes(2, 1024, 64, 32)
    assert index_full(L, ws_bytes=need - 1) == WORKSPACE


def test_index_reindex_rejects_bad_arguments(L):
    def call(**kw):
        a = dict(iq=FAKE, w=FAKE, ik=FAKE, N=FAKE, B=2, n_cap=1024, pool=FAKE, Lp=256, K=64,
                 topk=FAKE, ws=FAKE, ws_bytes=0)
        a.update(kw)
        return L.csa2_index_reindex(P(a["iq"]), P(a["w"]), P(a["ik"]), P(a["N"]), a["B"],
                                    a["n_cap"], P(a["pool"]), a["Lp"], a["K"], P(a["topk"]),
                                    P(a["ws"]), a["ws_bytes"], None, None)
    assert call(Lp=0) == INVALID
    assert call(pool=0) == INVALID
    assert call(Lp=40000) == UNSUPPORTED
    assert call(ws_bytes=csa2.index_reindex_workspace_bytes(2, 256, 64) - 8) == WORKSPACE


def test_attend_rejects_bad_arguments(L):
    def call(**kw):
        a = dict(mode=2, q=FAKE, scale=1.0, codes=FAKE, scales=FAKE, n_cap=1024, N=FAKE,
                 idx=FAKE, K=512, swa=FAKE, swa_scale=FAKE, swa_len=FAKE, W=128, B=8, out=FAKE,
                 lse=None, ws=FAKE, ws_bytes=0)
        a.update(kw)
        return L.csa2_attend(a["mode"], P(a["q"]), a["scale"], P(a["codes"]), P(a["scales"]),
                             a["n_cap"], P(a["N"]), P(a["idx"]), a["K"], P(a["swa"]),
                             P(a["swa_scale"]), P(a["swa_len"]), a["W"], a["B"], P(a["out"]),
                             P(a["lse"]), P(a["ws"]), a["ws_bytes"], None, None)
    assert call(mode=3) == INVALID
    assert call(mode=-1) == INVALID
    assert call(K=0) == INVALID
    assert call(W=-1) == INVALID
    assert call(q=MIS) == INVALID
    assert call(swa=0) == INVALID
    assert call(scale=float("nan")) == INVALID
    assert call(K=5000) == UNSUPPORTED
    assert call(ws_bytes=csa2.attend_workspace_bytes(8, 512, 128) - 1) == WORKSPACE


def test_calls_fail_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(csa2, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(csa2, "_lib", None)
    with pytest.raises(ImportError):
        csa2.lib()
