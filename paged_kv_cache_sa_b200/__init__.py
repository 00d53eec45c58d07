"""Page-sparse decode attention over a paged KV cache, for B200 (sm_100a).

Thin Python binding over the C ABI of ``lib/libsa.so`` (declared in ``include/sa.h``):
it only marshals torch tensors (device memory) and the current CUDA stream into the
library's plain pointers and sizes.  Every step of the computation runs in the
library's CUDA kernels; there is no Python or CPU fallback, and importing this
package fails loudly when the library has not been built.

Functions (all asynchronous on ``torch.cuda.current_stream()``):

  page_summaries(geom, k_cache, page_table, seq_lens, summ)
  update_summaries(geom, k_cache, page_table, seq_lens, summ, n_tail_pages=1)
  select_pages(geom, q, summ, page_table, seq_lens, budget, sink, window, ws, ...)
  sparse_decode(geom, q, k_cache, v_cache, summ, page_table, seq_lens, budget, sink,
                window, scale, out, lse, ws, ...)
  attend_selected(geom, q, k_cache, v_cache, page_table, seq_lens, sel, sel_count,
                  scale, out, lse, ws)
  prune_compact(geom, k_cache, v_cache, page_table, seq_lens, keep, free_pages, ...)

``Workspace`` owns one zero-initialised device buffer sized for a geometry.
"""

from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libsa.so")

SA_OK = 0
SA_ERR_INVALID_ARG, SA_ERR_UNSUPPORTED, SA_ERR_WORKSPACE = -1, -2, -3
STATUS = {0: "SA_OK", -1: "SA_ERR_INVALID_ARG", -2: "SA_ERR_UNSUPPORTED", -3: "SA_ERR_WORKSPACE",
          -4: "SA_ERR_CUDA", -5: "SA_ERR_DEVICE_CHECK", -6: "SA_ERR_TIMEOUT",
          -7: "SA_ERR_NO_SPACE"}

# every symbol include/sa.h declares
EXPORTS = ["sa_status_string", "sa_version", "sa_decode_workspace_size", "sa_prune_workspace_size",
           "sa_workspace_init", "sa_workspace_status", "sa_page_summaries", "sa_update_summaries",
           "sa_page_scores", "sa_select_pages", "sa_sparse_decode", "sa_attend_selected",
           "sa_prune_compact", "sa_sparse_decode_noalloc", "sa_summary_fp8_record_bytes",
           "sa_page_summaries_fp8", "sa_update_summaries_fp8", "sa_page_scores_fp8",
           "sa_sparse_decode_fp8", "sa_sparse_decode_fused"]


class SaError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__("%s failed: %s (%d)" % (what, STATUS.get(status, "?"), status))
        self.status = status


class sa_geom(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("B", "Hq", "Hkv", "Dk", "Dv", "P", "max_pages", "n_pool", "v_aliases_k")]


@dataclasses.dataclass
class Geometry:
    B: int
    Hq: int
    Hkv: int
    Dk: int
    Dv: int
    P: int
    max_pages: int
    n_pool: int
    v_aliases_k: int = 0

    def c(self) -> sa_geom:
        return sa_geom(self.B, self.Hq, self.Hkv, self.Dk, self.Dv, self.P, self.max_pages,
                       self.n_pool, self.v_aliases_k)

    @classmethod
    def of(cls, g) -> "Geometry":
        return cls(g.B, g.Hq, g.Hkv, g.Dk, g.Dv, g.P, g.max_pages, g.n_pool, g.v_aliases_k)


def _load(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError("libsa.so is not built (%s); run __graft_entry__.build() or "
                          "python paged_kv_cache_sa_b200/build.py" % path)
    lib = ctypes.CDLL(path)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    G = ctypes.POINTER(sa_geom)
    sig = {
        "sa_status_string": ([i32], ctypes.c_char_p),
        "sa_version": ([], i32),
        "sa_decode_workspace_size": ([G, i32], sz),
        "sa_prune_workspace_size": ([G], sz),
        "sa_workspace_init": ([vp, sz, vp], i32),
        "sa_workspace_status": ([vp, vp], i32),
        "sa_page_summaries": ([G, vp, vp, vp, vp, vp], i32),
        "sa_update_summaries": ([G, vp, vp, vp, i32, vp, vp], i32),
        "sa_page_scores": ([G, vp, vp, vp, vp, vp, vp, sz, vp], i32),
        "sa_select_pages": ([G, vp, vp, vp, vp, i32, i32, i32, vp, i32, vp, vp, vp, vp, vp, sz,
                             vp], i32),
        "sa_sparse_decode": ([G, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, ctypes.c_float, vp,
                              vp, vp, vp, vp, sz, vp], i32),
        "sa_sparse_decode_fused": ([G, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32,
                                    ctypes.c_float, vp, vp, vp, vp, vp, sz, vp], i32),
        "sa_sparse_decode_noalloc": ([G, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32,
                                      ctypes.c_float, vp, vp, vp, vp, vp, vp], i32),
        "sa_summary_fp8_record_bytes": ([G], sz),
        "sa_page_summaries_fp8": ([G, vp, vp, vp, vp, vp], i32),
        "sa_update_summaries_fp8": ([G, vp, vp, vp, i32, vp, vp], i32),
        "sa_page_scores_fp8": ([G, vp, vp, vp, vp, vp, vp, sz, vp], i32),
        "sa_sparse_decode_fp8": ([G, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, ctypes.c_float,
                                  vp, vp, vp, vp, vp, sz, vp], i32),
        "sa_attend_selected": ([G, vp, vp, vp, vp, vp, vp, vp, vp, i32, ctypes.c_float, vp, vp,
                                vp, sz, vp], i32),
        "sa_prune_compact": ([G, vp, vp, vp, vp, vp, vp, i64, vp, vp, vp, vp, vp, vp, vp, vp, sz,
                              vp], i32),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    return lib


lib = _load()


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(st: int, what: str):
    if st != SA_OK:
        raise SaError(st, what)


def decode_workspace_size(geom: Geometry, budget: int) -> int:
    g = geom.c()
    return int(lib.sa_decode_workspace_size(ctypes.byref(g), int(budget)))


def prune_workspace_size(geom: Geometry) -> int:
    g = geom.c()
    return int(lib.sa_prune_workspace_size(ctypes.byref(g)))


class Workspace:
    """A zero-initialised device buffer for one stream's calls."""

    def __init__(self, nbytes: int, device=None, stream=None):
        if nbytes <= 0:
            raise ValueError("workspace size must be positive (invalid geometry?)")
        self.buf = torch.empty(int(nbytes), dtype=torch.uint8, device=device or "cuda")
        self.nbytes = int(nbytes)
        _check(lib.sa_workspace_init(_ptr(self.buf), self.nbytes, _stream(stream)),
               "sa_workspace_init")

    @classmethod
    def for_decode(cls, geom: Geometry, budget: int, **kw) -> "Workspace":
        return cls(decode_workspace_size(geom, budget), **kw)

    @classmethod
    def for_prune(cls, geom: Geometry, **kw) -> "Workspace":
        return cls(prune_workspace_size(geom), **kw)

    def status(self, stream=None) -> int:
        """Synchronise the stream and return (and clear) the device status word."""
        return int(lib.sa_workspace_status(_ptr(self.buf), _stream(stream)))


def page_summaries(geom: Geometry, k_cache, page_table, seq_lens, summ, stream=None):
    g = geom.c()
    _check(lib.sa_page_summaries(ctypes.byref(g), _ptr(k_cache), _ptr(page_table), _ptr(seq_lens),
                                 _ptr(summ), _stream(stream)), "sa_page_summaries")
    return summ


def update_summaries(geom: Geometry, k_cache, page_table, seq_lens, summ, n_tail_pages: int = 1,
                     stream=None):
    g = geom.c()
    _check(lib.sa_update_summaries(ctypes.byref(g), _ptr(k_cache), _ptr(page_table),
                                   _ptr(seq_lens), int(n_tail_pages), _ptr(summ),
                                   _stream(stream)), "sa_update_summaries")
    return summ


def page_scores(geom: Geometry, q, summ, page_table, seq_lens, ws: Workspace, scores=None,
                stream=None):
    """Page scores alone: [B][Hkv][max_pages] fp32 (-inf past each sequence's pages)."""
    if scores is None:
        scores = torch.empty((geom.B, geom.Hkv, geom.max_pages), dtype=torch.float32,
                             device=q.device)
    g = geom.c()
    _check(lib.sa_page_scores(ctypes.byref(g), _ptr(q), _ptr(summ), _ptr(page_table),
                              _ptr(seq_lens), _ptr(scores), _ptr(ws.buf), ws.nbytes,
                              _stream(stream)), "sa_page_scores")
    return scores


def select_pages(geom: Geometry, q, summ, page_table, seq_lens, budget, sink, window,
                 ws: Workspace, sel=None, sel_count=None, scores=None, k_cache=None,
                 n_tail_refresh: int = 0, sel_phys=None, stream=None):
    """Score every page and select the top pages (plus sink and window pages).
    With ``n_tail_refresh`` > 0 the last pages' summaries are first recomputed from
    ``k_cache`` (the decode-time update after an append)."""
    K = budget // geom.P
    dev = q.device
    if sel is None:
        sel = torch.empty((geom.B, geom.Hkv, K), dtype=torch.int32, device=dev)
    if sel_count is None:
        sel_count = torch.empty((geom.B, geom.Hkv), dtype=torch.int32, device=dev)
    g = geom.c()
    _check(lib.sa_select_pages(ctypes.byref(g), _ptr(q), _ptr(summ), _ptr(page_table),
                               _ptr(seq_lens), int(budget), int(sink), int(window),
                               _ptr(k_cache), int(n_tail_refresh), _ptr(sel), _ptr(sel_count),
                               _ptr(sel_phys), _ptr(scores), _ptr(ws.buf), ws.nbytes,
                               _stream(stream)),
           "sa_select_pages")
    return sel, sel_count


def sparse_decode(geom: Geometry, q, k_cache, v_cache, summ, page_table, seq_lens, budget, sink,
                  window, scale, ws: Workspace, out=None, lse=None, sel_out=None,
                  sel_count_out=None, n_tail_refresh: int = 0, stream=None):
    dev = q.device
    if out is None:
        out = torch.empty((geom.B, geom.Hq, geom.Dv), dtype=torch.float32, device=dev)
    if lse is None:
        lse = torch.empty((geom.B, geom.Hq), dtype=torch.float32, device=dev)
    g = geom.c()
    _check(lib.sa_sparse_decode(ctypes.byref(g), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(summ),
                                _ptr(page_table), _ptr(seq_lens), int(budget), int(sink),
                                int(window), int(n_tail_refresh), float(scale), _ptr(out),
                                _ptr(lse), _ptr(sel_out), _ptr(sel_count_out), _ptr(ws.buf),
                                ws.nbytes, _stream(stream)), "sa_sparse_decode")
    return out, lse


def sparse_decode_fused(geom: Geometry, q, k_cache, v_cache, summ, page_table, seq_lens, budget,
                        sink, window, scale, ws: Workspace, out=None, lse=None, sel_out=None,
                        sel_count_out=None, n_tail_refresh: int = 0, stream=None):
    """sparse_decode in one persistent launch (grouped-query geometry)."""
    dev = q.device
    if out is None:
        out = torch.empty((geom.B, geom.Hq, geom.Dv), dtype=torch.float32, device=dev)
    if lse is None:
        lse = torch.empty((geom.B, geom.Hq), dtype=torch.float32, device=dev)
    g = geom.c()
    _check(lib.sa_sparse_decode_fused(ctypes.byref(g), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                      _ptr(summ), _ptr(page_table), _ptr(seq_lens), int(budget),
                                      int(sink), int(window), int(n_tail_refresh),
                                      float(scale), _ptr(out), _ptr(lse), _ptr(sel_out),
                                      _ptr(sel_count_out), _ptr(ws.buf), ws.nbytes,
                                      _stream(stream)), "sa_sparse_decode_fused")
    return out, lse


def summary_fp8_record_bytes(geom: Geometry) -> int:
    g = geom.c()
    return int(lib.sa_summary_fp8_record_bytes(ctypes.byref(g)))


def empty_summaries_fp8(geom: Geometry, device=None) -> torch.Tensor:
    """A zeroed fp8 record buffer [n_pool, Hkv, 2*Dk + 16] uint8."""
    n = summary_fp8_record_bytes(geom)
    if n == 0:
        raise SaError(SA_ERR_UNSUPPORTED, "fp8 summaries")
    return torch.zeros((geom.n_pool, geom.Hkv, n), dtype=torch.uint8, device=device or "cuda")


def page_summaries_fp8(geom: Geometry, k_cache, page_table, seq_lens, summ8, stream=None):
    g = geom.c()
    _check(lib.sa_page_summaries_fp8(ctypes.byref(g), _ptr(k_cache), _ptr(page_table),
                                     _ptr(seq_lens), _ptr(summ8), _stream(stream)),
           "sa_page_summaries_fp8")
    return summ8


def update_summaries_fp8(geom: Geometry, k_cache, page_table, seq_lens, summ8,
                         n_tail_pages: int = 1, stream=None):
    g = geom.c()
    _check(lib.sa_update_summaries_fp8(ctypes.byref(g), _ptr(k_cache), _ptr(page_table),
                                       _ptr(seq_lens), int(n_tail_pages), _ptr(summ8),
                                       _stream(stream)), "sa_update_summaries_fp8")
    return summ8


def page_scores_fp8(geom: Geometry, q, summ8, page_table, seq_lens, ws: Workspace, scores=None,
                    stream=None):
    if scores is None:
        scores = torch.empty((geom.B, geom.Hkv, geom.max_pages), dtype=torch.float32,
                             device=q.device)
    g = geom.c()
    _check(lib.sa_page_scores_fp8(ctypes.byref(g), _ptr(q), _ptr(summ8), _ptr(page_table),
                                  _ptr(seq_lens), _ptr(scores), _ptr(ws.buf), ws.nbytes,
                                  _stream(stream)), "sa_page_scores_fp8")
    return scores


def sparse_decode_fp8(geom: Geometry, q, k_cache, v_cache, summ8, page_table, seq_lens, budget,
                      sink, window, scale, ws: Workspace, out=None, lse=None, sel_out=None,
                      sel_count_out=None, n_tail_refresh: int = 0, stream=None):
    dev = q.device
    if out is None:
        out = torch.empty((geom.B, geom.Hq, geom.Dv), dtype=torch.float32, device=dev)
    if lse is None:
        lse = torch.empty((geom.B, geom.Hq), dtype=torch.float32, device=dev)
    g = geom.c()
    _check(lib.sa_sparse_decode_fp8(ctypes.byref(g), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                    _ptr(summ8), _ptr(page_table), _ptr(seq_lens), int(budget),
                                    int(sink), int(window), int(n_tail_refresh), float(scale),
                                    _ptr(out), _ptr(lse), _ptr(sel_out), _ptr(sel_count_out),
                                    _ptr(ws.buf), ws.nbytes, _stream(stream)),
           "sa_sparse_decode_fp8")
    return out, lse


def sparse_decode_noalloc(geom: Geometry, q, k_cache, v_cache, summ, page_table, seq_lens,
                          budget, sink, window, scale, out=None, lse=None, sel_out=None,
                          sel_count_out=None, status_out=None, n_tail_refresh: int = 0,
                          stream=None):
    """sa_sparse_decode on the library's static scratch (no workspace argument)."""
    dev = q.device
    if out is None:
        out = torch.empty((geom.B, geom.Hq, geom.Dv), dtype=torch.float32, device=dev)
    if lse is None:
        lse = torch.empty((geom.B, geom.Hq), dtype=torch.float32, device=dev)
    g = geom.c()
    _check(lib.sa_sparse_decode_noalloc(ctypes.byref(g), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                        _ptr(summ), _ptr(page_table), _ptr(seq_lens), int(budget),
                                        int(sink), int(window), int(n_tail_refresh), float(scale),
                                        _ptr(out), _ptr(lse), _ptr(sel_out), _ptr(sel_count_out),
                                        _ptr(status_out), _stream(stream)),
           "sa_sparse_decode_noalloc")
    return out, lse


def attend_selected(geom: Geometry, q, k_cache, v_cache, page_table, seq_lens, sel, sel_count,
                    scale, ws: Workspace, out=None, lse=None, sel_phys=None, stream=None):
    dev = q.device
    if out is None:
        out = torch.empty((geom.B, geom.Hq, geom.Dv), dtype=torch.float32, device=dev)
    if lse is None:
        lse = torch.empty((geom.B, geom.Hq), dtype=torch.float32, device=dev)
    g = geom.c()
    _check(lib.sa_attend_selected(ctypes.byref(g), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                  _ptr(page_table), _ptr(seq_lens), _ptr(sel), _ptr(sel_count),
                                  _ptr(sel_phys), int(sel.shape[-1]), float(scale), _ptr(out),
                                  _ptr(lse),
                                  _ptr(ws.buf), ws.nbytes, _stream(stream)), "sa_attend_selected")
    return out, lse


def prune_compact(geom: Geometry, k_cache, v_cache, page_table, seq_lens, keep, free_pages,
                  k_dst, v_dst, summ, ws: Workspace, new_page_table=None, new_seq_lens=None,
                  pos_map=None, logical_len=None, stream=None):
    dev = k_cache.device
    width = geom.max_pages * geom.P
    if new_page_table is None:
        new_page_table = torch.empty((geom.B, geom.max_pages), dtype=torch.int32, device=dev)
    if new_seq_lens is None:
        new_seq_lens = torch.empty((geom.B,), dtype=torch.int32, device=dev)
    if pos_map is None:
        pos_map = torch.empty((geom.B, width), dtype=torch.int32, device=dev)
    if logical_len is None:
        logical_len = torch.empty((geom.B,), dtype=torch.int32, device=dev)
    g = geom.c()
    _check(lib.sa_prune_compact(ctypes.byref(g), _ptr(k_cache), _ptr(v_cache), _ptr(page_table),
                                _ptr(seq_lens), _ptr(keep), _ptr(free_pages),
                                int(free_pages.numel()), _ptr(k_dst), _ptr(v_dst), _ptr(summ),
                                _ptr(new_page_table), _ptr(new_seq_lens), _ptr(pos_map),
                                _ptr(logical_len), _ptr(ws.buf), ws.nbytes, _stream(stream)),
           "sa_prune_compact")
    return new_page_table, new_seq_lens, pos_map, logical_len
