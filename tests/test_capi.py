"""The C-ABI library builds, loads without a GPU, and exports exactly what
include/sa.h declares (the traced build: sa.h and include/sa_trace.h); the CPU-only host
logic of the binding."""

import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared(header="sa.h"):
    src = open(os.path.join(ROOT, "include", header)).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sa_[a-z0-9_]+)\s*\(", src)))


def _build(**kw):
    # build.py by path: importing the package first would load a possibly stale library
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_sa_build", os.path.join(ROOT, "paged_kv_cache_sa_b200", "build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    return b.build(**kw)


def _exported(path):
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True,
                         text=True).stdout
    return sorted({ln.split()[-1] for ln in out.splitlines()
                   if ln.split() and ln.split()[-1].startswith("sa_")})


@pytest.fixture(scope="module")
def libpath():
    return _build()


def test_header_declares_the_expected_entry_points():
    decl = _declared()
    for name in ("sa_page_summaries", "sa_update_summaries", "sa_select_pages",
                 "sa_sparse_decode", "sa_attend_selected", "sa_prune_compact",
                 "sa_decode_workspace_size", "sa_prune_workspace_size", "sa_workspace_init",
                 "sa_workspace_status", "sa_status_string", "sa_version", "sa_page_scores",
                 "sa_sparse_decode_noalloc", "sa_summary_fp8_record_bytes",
                 "sa_page_summaries_fp8", "sa_update_summaries_fp8", "sa_page_scores_fp8",
                 "sa_sparse_decode_fp8"):
        assert name in decl


def test_library_exports_every_declared_symbol(libpath):
    lib = ctypes.CDLL(libpath)
    for name in _declared():
        assert hasattr(lib, name), name
    assert _exported(libpath) == _declared()


def test_every_header_is_covered():
    assert sorted(os.listdir(os.path.join(ROOT, "include"))) == ["sa.h", "sa_trace.h"]


def test_traced_library_exports_sa_h_and_sa_trace_h():
    """The phase-timeline build: everything libsa.so exports plus sa_trace_set."""
    path = _build(trace=True)
    lib = ctypes.CDLL(path)
    want = sorted(set(_declared()) | set(_declared("sa_trace.h")))
    assert _declared("sa_trace.h") == ["sa_trace_set"]
    for name in want:
        assert hasattr(lib, name), name
    assert _exported(path) == want


def test_binding_loads_and_sizes_workspaces(libpath):
    import paged_kv_cache_sa_b200 as sa
    for name in sa.EXPORTS:
        assert hasattr(sa.lib, name)
    assert sa.lib.sa_version() >= 10000
    assert sa.lib.sa_status_string(-7) == b"not enough free pages"
    g = sa.Geometry(B=8, Hq=32, Hkv=8, Dk=128, Dv=128, P=16, max_pages=2048, n_pool=16384)
    n = sa.decode_workspace_size(g, 2048)
    # header + scores + selection + counts + split partials
    assert n >= 256 + 8 * 8 * 2048 * 4 + 8 * 8 * 128 * 4
    assert sa.decode_workspace_size(g, 2004) == 0            # budget not a multiple of P
    bad = sa.Geometry(B=8, Hq=32, Hkv=8, Dk=96, Dv=96, P=16, max_pages=2048, n_pool=16384)
    assert sa.decode_workspace_size(bad, 2048) == 0          # unsupported head dim
    assert sa.prune_workspace_size(g) > 256


def test_fp8_record_size_and_host_checks(libpath):
    import paged_kv_cache_sa_b200 as sa
    g = sa.Geometry(B=8, Hq=32, Hkv=8, Dk=128, Dv=128, P=16, max_pages=2048, n_pool=16384)
    assert sa.summary_fp8_record_bytes(g) == 2 * 128 + 16
    g64 = sa.Geometry(B=2, Hq=32, Hkv=4, Dk=64, Dv=64, P=16, max_pages=64, n_pool=128)
    assert sa.summary_fp8_record_bytes(g64) == 2 * 64 + 16
    lat = sa.Geometry(B=2, Hq=128, Hkv=1, Dk=576, Dv=512, P=64, max_pages=64, n_pool=128,
                      v_aliases_k=1)
    assert sa.summary_fp8_record_bytes(lat) == 0
    # argument errors come back before any CUDA call
    c = lat.c()
    dummy = ctypes.c_void_p(4096)
    assert sa.lib.sa_page_summaries_fp8(ctypes.byref(c), dummy, dummy, dummy, dummy,
                                        None) == sa.SA_ERR_UNSUPPORTED
    c = g.c()
    assert sa.lib.sa_page_summaries_fp8(ctypes.byref(c), None, dummy, dummy, dummy,
                                        None) == sa.SA_ERR_INVALID_ARG
    assert sa.lib.sa_sparse_decode_fp8(ctypes.byref(c), dummy, dummy, dummy, dummy, dummy, dummy,
                                       2048, 64, 512, 0, 0.1, dummy, dummy, None, None, dummy,
                                       16, None) == sa.SA_ERR_WORKSPACE
    assert sa.lib.sa_sparse_decode_fp8(ctypes.byref(c), dummy, dummy, dummy, dummy, dummy, dummy,
                                       2048, 64, 3000, 0, 0.1, dummy, dummy, None, None, dummy,
                                       1 << 30, None) == sa.SA_ERR_INVALID_ARG


def test_no_cpu_fallback_in_binding():
    src = open(os.path.join(ROOT, "paged_kv_cache_sa_b200", "__init__.py")).read()
    assert "import oracle" not in src and "from oracle" not in src
    assert "numpy" not in src


def test_argument_errors_before_any_launch(libpath):
    """Every decode, selection, attention and compaction entry point rejects bad geometry,
    budgets, pointers, alignment and workspaces with the status include/sa.h documents,
    before any CUDA call (so this runs without a GPU)."""
    import paged_kv_cache_sa_b200 as sa
    lib = sa.lib
    A = ctypes.c_void_p(1 << 20)          # aligned dummy device address, never touched
    MIS = ctypes.c_void_p((1 << 20) + 4)  # not 16-byte aligned
    INV, UNS, WSE = sa.SA_ERR_INVALID_ARG, sa.SA_ERR_UNSUPPORTED, sa.SA_ERR_WORKSPACE
    good = sa.Geometry(B=2, Hq=8, Hkv=2, Dk=128, Dv=128, P=16, max_pages=64, n_pool=256)
    big_ws = 1 << 30

    def geom(**kw):
        d = dict(good.__dict__)
        d.update(kw)
        return sa.Geometry(**d).c()

    def decode(fn=lib.sa_sparse_decode, g=None, q=A, v=A, budget=512, sink=16, window=64,
               tail=0, ws=A, ws_bytes=big_ws):
        c = g if g is not None else good.c()
        return fn(ctypes.byref(c), q, A, v, A, A, A, budget, sink, window, tail, 0.1, A, A,
                  None, None, ws, ws_bytes, None)

    assert lib.sa_sparse_decode(None, A, A, A, A, A, A, 512, 16, 64, 0, 0.1, A, A, None, None,
                                A, big_ws, None) == INV
    for fn in (lib.sa_sparse_decode, lib.sa_sparse_decode_fused):
        assert decode(fn, g=geom(B=0)) == INV                    # empty batch
        assert decode(fn, g=geom(Hq=9)) == INV                   # Hq not a multiple of Hkv
        assert decode(fn, g=geom(P=8)) == UNS                    # page size
        assert decode(fn, g=geom(Dk=96, Dv=96)) == UNS           # head dim
        assert decode(fn, g=geom(Hq=32, Hkv=2)) == UNS           # 16 query heads per KV head
        assert decode(fn, budget=500) == INV                     # budget not a multiple of P
        assert decode(fn, budget=0) == INV
        assert decode(fn, sink=-16) == INV
        assert decode(fn, sink=8) == INV                         # sink not a multiple of P
        assert decode(fn, sink=256, window=272) == INV           # sink + window > budget
        assert decode(fn, q=None) == INV
        assert decode(fn, v=None) == INV                         # separate V needed
        assert decode(fn, q=MIS) == INV                          # 16-byte alignment
        assert decode(fn, tail=17) == INV                        # refresh at most 16 pages
        assert decode(fn, tail=-1) == INV
        assert decode(fn, g=geom(max_pages=60000)) == UNS        # page-table row > 200 KB
        assert decode(fn, ws=None) == WSE
        assert decode(fn, ws=MIS) == WSE
        assert decode(fn, ws_bytes=1024) == WSE
    # the single launch takes the grouped-query geometry only
    lat = sa.Geometry(B=2, Hq=128, Hkv=1, Dk=576, Dv=512, P=64, max_pages=64, n_pool=256,
                      v_aliases_k=1).c()
    assert decode(lib.sa_sparse_decode_fused, g=lat, budget=2048, sink=64, window=512) == UNS

    # selection: outputs required, and K to refresh from
    c = good.c()
    assert lib.sa_select_pages(ctypes.byref(c), A, A, A, A, 512, 16, 64, None, 0, None, A,
                               None, None, A, big_ws, None) == INV
    assert lib.sa_select_pages(ctypes.byref(c), A, A, A, A, 512, 16, 64, None, 1, A, A,
                               None, None, A, big_ws, None) == INV
    assert lib.sa_select_pages(ctypes.byref(c), A, A, A, A, 512, 16, 64, A, 0, A, A,
                               None, None, A, 64, None) == WSE

    # attention over a given selection: stride 1..65536
    for stride in (0, 65537):
        assert lib.sa_attend_selected(ctypes.byref(c), A, A, A, A, A, A, A, None, stride, 0.1,
                                      A, A, A, big_ws, None) == INV
    assert lib.sa_attend_selected(ctypes.byref(c), A, A, None, A, A, A, A, None, 32, 0.1,
                                  A, A, A, big_ws, None) == INV

    # compaction: free-page list, V buffers, workspace
    def prune(n_free=4, free=A, v_dst=A, ws_bytes=big_ws):
        return lib.sa_prune_compact(ctypes.byref(c), A, A, A, A, A, free, n_free, A, v_dst, A,
                                    A, A, A, A, A, ws_bytes, None)
    assert prune(n_free=-1) == INV
    assert prune(free=None) == INV
    assert prune(v_dst=None) == INV
    assert prune(ws_bytes=16) == WSE

    # the static scratch of the allocation-free call does not hold the latent geometry at
    # 16 sequences of 64K tokens with budget 2048 (about 38 MB)
    lat16 = sa.Geometry(B=16, Hq=128, Hkv=1, Dk=576, Dv=512, P=64, max_pages=1024,
                        n_pool=16384, v_aliases_k=1)
    assert sa.decode_workspace_size(lat16, 2048) > (32 << 20)
    c16 = lat16.c()
    assert lib.sa_sparse_decode_noalloc(ctypes.byref(c16), A, A, None, A, A, A, 2048, 64, 512,
                                        0, 0.1, A, A, None, None, None, None) == WSE
