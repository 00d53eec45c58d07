"""CPU oracle for page-sparse decode and prefix-cache pruning (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
may import this package.  The product library never does, and this package
never touches the CUDA library.  The arithmetic lives in ``sa_oracle.c`` (plain
C, fp64, one loop per definition); this module only builds it with gcc and
marshals numpy arrays through ctypes.

Every function is pinned by ``tests/test_oracle_pins.py`` against closed forms,
library routines (numpy / scipy), invariants and brute force.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sa_oracle.c")
_LIB = os.path.join(_HERE, "lib", "libsa_oracle.so")

__all__ = ["build", "load", "page_summaries", "page_scores", "select_pages", "attend",
           "dense_attend", "prune_compact", "decode", "e4m3_values", "e4m3_outward",
           "page_summaries_fp8", "page_scores_fp8", "decode_fp8"]


class _Geom(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("B", "Hq", "Hkv", "Dk", "Dv", "P", "max_pages", "n_pool", "v_aliases_k")]


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/lib/libsa_oracle.so`` (gcc, -O2, no fast-math)."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    os.makedirs(os.path.dirname(_LIB), exist_ok=True)
    tmp = _LIB + ".tmp.%d" % os.getpid()
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
                           "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
    os.replace(tmp, _LIB)
    return _LIB


_lib = None


def load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i32 = ctypes.c_int32
        lib.oracle_page_summaries.argtypes = [ctypes.POINTER(_Geom), P, P, P, P]
        lib.oracle_page_summaries.restype = None
        lib.oracle_page_scores.argtypes = [ctypes.POINTER(_Geom), P, P, P, P, P]
        lib.oracle_page_scores.restype = None
        lib.oracle_select_pages.argtypes = [ctypes.POINTER(_Geom), P, P, i32, i32, i32, P, P]
        lib.oracle_select_pages.restype = ctypes.c_int
        lib.oracle_attend.argtypes = [ctypes.POINTER(_Geom), P, P, P, P, P, P, P, i32,
                                      ctypes.c_double, P, P]
        lib.oracle_attend.restype = None
        lib.oracle_dense_attend.argtypes = [i32, i32, i32, i32, P, P, P, ctypes.c_double, P, P]
        lib.oracle_dense_attend.restype = None
        lib.oracle_prune_compact.argtypes = [ctypes.POINTER(_Geom), P, P, P, P, P, P,
                                             ctypes.c_int64, P, P, P, P, P, P, P]
        lib.oracle_prune_compact.restype = ctypes.c_int64
        lib.oracle_e4m3_values.argtypes = [P]
        lib.oracle_e4m3_values.restype = None
        lib.oracle_e4m3_outward.argtypes = [ctypes.c_double, i32]
        lib.oracle_e4m3_outward.restype = ctypes.c_uint8
        lib.oracle_encode_fp8.argtypes = [ctypes.POINTER(_Geom), P, P, P, P]
        lib.oracle_encode_fp8.restype = None
        lib.oracle_page_scores_fp8.argtypes = [ctypes.POINTER(_Geom), P, P, P, P, P]
        lib.oracle_page_scores_fp8.restype = None
        _lib = lib
    return _lib


def _geom(g) -> _Geom:
    return _Geom(g.B, g.Hq, g.Hkv, g.Dk, g.Dv, g.P, g.max_pages, g.n_pool, g.v_aliases_k)


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def page_summaries(geom, k_cache, page_table, seq_lens, summ=None) -> np.ndarray:
    """summ [n_pool, Hkv, 2, Dk] bf16 bits (row 0 min, row 1 max); untouched pages 0."""
    k_cache = _c(k_cache, np.uint16)
    pt, sl = _c(page_table, np.int32), _c(seq_lens, np.int32)
    if summ is None:
        summ = np.zeros((geom.n_pool, geom.Hkv, 2, geom.Dk), dtype=np.uint16)
    g = _geom(geom)
    load().oracle_page_summaries(ctypes.byref(g), _p(k_cache), _p(pt), _p(sl), _p(summ))
    return summ


def page_scores(geom, q, summ, page_table, seq_lens) -> np.ndarray:
    """scores [B, Hkv, max_pages] float64 (-inf beyond each sequence's pages)."""
    q, summ = _c(q, np.uint16), _c(summ, np.uint16)
    pt, sl = _c(page_table, np.int32), _c(seq_lens, np.int32)
    out = np.empty((geom.B, geom.Hkv, geom.max_pages), dtype=np.float64)
    g = _geom(geom)
    load().oracle_page_scores(ctypes.byref(g), _p(q), _p(summ), _p(pt), _p(sl), _p(out))
    return out


def e4m3_values() -> np.ndarray:
    """Value of each of the 256 FP8 E4M3 codes (NaN for 0x7F and 0xFF)."""
    out = np.empty(256, dtype=np.float64)
    load().oracle_e4m3_values(_p(out))
    return out


def e4m3_outward(x: float, up: bool) -> int:
    """Tightest finite E4M3 code >= x (up) or <= x (down); zero is 0x00."""
    return int(load().oracle_e4m3_outward(float(x), 1 if up else 0))


def page_summaries_fp8(geom, k_cache, page_table, seq_lens) -> np.ndarray:
    """fp8 records [n_pool, Hkv, 2*Dk + 16] uint8 of every used page: Dk codes of the
    min row (rounded toward -inf), Dk codes of the max row (toward +inf), the int8
    exponent e, 15 zero bytes; values = code * 2^e.  Untouched pages are 0."""
    summ = page_summaries(geom, k_cache, page_table, seq_lens)
    out = np.zeros((geom.n_pool, geom.Hkv, 2 * geom.Dk + 16), dtype=np.uint8)
    pt, sl = _c(page_table, np.int32), _c(seq_lens, np.int32)
    g = _geom(geom)
    load().oracle_encode_fp8(ctypes.byref(g), _p(summ), _p(pt), _p(sl), _p(out))
    return out


def page_scores_fp8(geom, q, summ8, page_table, seq_lens) -> np.ndarray:
    """The page bound over decoded fp8 records: [B, Hkv, max_pages] float64."""
    q, summ8 = _c(q, np.uint16), _c(summ8, np.uint8)
    pt, sl = _c(page_table, np.int32), _c(seq_lens, np.int32)
    out = np.empty((geom.B, geom.Hkv, geom.max_pages), dtype=np.float64)
    g = _geom(geom)
    load().oracle_page_scores_fp8(ctypes.byref(g), _p(q), _p(summ8), _p(pt), _p(sl), _p(out))
    return out


def select_pages(geom, scores, seq_lens, budget, sink, window):
    """(sel [B, Hkv, budget/P] int32 ascending, -1 padded;  sel_count [B, Hkv] int32)."""
    K = budget // geom.P
    scores = _c(scores, np.float64)
    sl = _c(seq_lens, np.int32)
    sel = np.empty((geom.B, geom.Hkv, K), dtype=np.int32)
    cnt = np.empty((geom.B, geom.Hkv), dtype=np.int32)
    g = _geom(geom)
    rc = load().oracle_select_pages(ctypes.byref(g), _p(scores), _p(sl), budget, sink, window,
                                    _p(sel), _p(cnt))
    if rc != 0:
        raise ValueError("invalid budget/sink/window for page size %d" % geom.P)
    return sel, cnt


def attend(geom, q, k_cache, v_cache, page_table, seq_lens, sel, sel_count, scale):
    """(out [B, Hq, Dv] float64, lse [B, Hq] float64) over the selected pages."""
    q, k_cache = _c(q, np.uint16), _c(k_cache, np.uint16)
    v_cache = None if v_cache is None else _c(v_cache, np.uint16)
    pt, sl = _c(page_table, np.int32), _c(seq_lens, np.int32)
    sel, sel_count = _c(sel, np.int32), _c(sel_count, np.int32)
    K = sel.shape[-1]
    out = np.empty((geom.B, geom.Hq, geom.Dv), dtype=np.float64)
    lse = np.empty((geom.B, geom.Hq), dtype=np.float64)
    g = _geom(geom)
    load().oracle_attend(ctypes.byref(g), _p(q), _p(k_cache), _p(v_cache), _p(pt), _p(sl),
                         _p(sel), _p(sel_count), K, float(scale), _p(out), _p(lse))
    return out, lse


def dense_attend(q, k, v, scale):
    """Dense softmax attention on contiguous arrays: q [G, Dk], k [L, Dk], v [L, Dv]."""
    q, k, v = _c(q, np.uint16), _c(k, np.uint16), _c(v, np.uint16)
    G, Dk = q.shape
    L, Dv = v.shape
    out = np.empty((G, Dv), dtype=np.float64)
    lse = np.empty((G,), dtype=np.float64)
    load().oracle_dense_attend(L, Dk, Dv, G, _p(q), _p(k), _p(v), float(scale), _p(out), _p(lse))
    return out, lse


def prune_compact(geom, k_cache, v_cache, page_table, seq_lens, keep, free_pages,
                  k_dst=None, v_dst=None, summ=None):
    """Compaction of kept tokens into fresh pages.

    Returns a dict with k_dst, v_dst, summ, new_page_table, new_seq_lens, pos_map,
    logical_len and pages_used; raises ValueError when free_pages is too short.
    k_dst / v_dst default to copies of the source pools.
    """
    k_cache = _c(k_cache, np.uint16)
    v_cache = None if v_cache is None else _c(v_cache, np.uint16)
    pt, sl = _c(page_table, np.int32), _c(seq_lens, np.int32)
    keep, free_pages = _c(keep, np.uint8), _c(free_pages, np.int32)
    k_dst = k_cache.copy() if k_dst is None else k_dst
    v_dst = (None if v_cache is None else v_cache.copy()) if v_dst is None else v_dst
    if summ is None:
        summ = np.zeros((geom.n_pool, geom.Hkv, 2, geom.Dk), dtype=np.uint16)
    width = geom.max_pages * geom.P
    npt = np.empty((geom.B, geom.max_pages), dtype=np.int32)
    nsl = np.empty((geom.B,), dtype=np.int32)
    pos = np.empty((geom.B, width), dtype=np.int32)
    ll = np.empty((geom.B,), dtype=np.int32)
    g = _geom(geom)
    used = load().oracle_prune_compact(ctypes.byref(g), _p(k_cache), _p(v_cache), _p(pt), _p(sl),
                                       _p(keep), _p(free_pages), int(free_pages.shape[0]),
                                       _p(k_dst), _p(v_dst), _p(summ), _p(npt), _p(nsl), _p(pos),
                                       _p(ll))
    if used < 0:
        raise ValueError("not enough free pages")
    return dict(k_dst=k_dst, v_dst=v_dst, summ=summ, new_page_table=npt, new_seq_lens=nsl,
                pos_map=pos, logical_len=ll, pages_used=int(used))


def decode(case, sel=None, sel_count=None):
    """The whole path on one ``synth.DecodeCase``: summaries -> scores -> selection ->
    attention.  Pass ``sel``/``sel_count`` to attend over a given selection instead.
    Returns a dict with summ, scores, sel, sel_count, out, lse."""
    g = case.geom
    summ = page_summaries(g, case.k_cache, case.page_table, case.seq_lens)
    scores = page_scores(g, case.q, summ, case.page_table, case.seq_lens)
    osel, ocnt = select_pages(g, scores, case.seq_lens, case.budget, case.sink, case.window)
    if sel is None:
        sel, sel_count = osel, ocnt
    out, lse = attend(g, case.q, case.k_cache, case.v_cache, case.page_table, case.seq_lens,
                      sel, sel_count, case.scale)
    return dict(summ=summ, scores=scores, sel=osel, sel_count=ocnt, out=out, lse=lse,
                attend_sel=sel, attend_count=sel_count)


def decode_fp8(case, sel=None, sel_count=None):
    """``decode`` with the page bound taken over fp8 summaries rounded outward
    (page_summaries_fp8 / page_scores_fp8); attention still reads the bf16 K and V."""
    g = case.geom
    summ8 = page_summaries_fp8(g, case.k_cache, case.page_table, case.seq_lens)
    scores = page_scores_fp8(g, case.q, summ8, case.page_table, case.seq_lens)
    osel, ocnt = select_pages(g, scores, case.seq_lens, case.budget, case.sink, case.window)
    if sel is None:
        sel, sel_count = osel, ocnt
    out, lse = attend(g, case.q, case.k_cache, case.v_cache, case.page_table, case.seq_lens,
                      sel, sel_count, case.scale)
    return dict(summ8=summ8, scores=scores, sel=osel, sel_count=ocnt, out=out, lse=lse,
                attend_sel=sel, attend_count=sel_count)
