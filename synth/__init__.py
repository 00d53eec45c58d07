"""Seeded synthetic inputs for query-aware page-sparse decode over a paged KV cache.

This module only *builds inputs*: bf16 query/key/value tensors, page tables,
sequence lengths and keep-masks, shaped like the long-context agent workloads
the source pages describe (multi-turn agent traces, SCBench-style shared
contexts of ~100K+ tokens).  None of those datasets is present, so every tensor
here is drawn from a seeded generator.  It holds none of the method's
arithmetic (no summaries, scores, selection, attention or compaction); both the
CPU oracle and the CUDA path consume what it returns.

Random numbers come from numpy's PCG64 seeded through ``SeedSequence([seed,
stream])``, one stream per tensor (``SeedSequence([seed, stream, chunk])`` per block
of 2^22 values for the large normal tensors, so that the blocks can be drawn on
several host threads with the same result), and are rounded to bf16 with
round-to-nearest-even.  bf16 tensors are returned as ``uint16`` bit patterns.

Workloads (sizes as named by the method's target configurations):

* ``tiny``      - 1 x 4096 tokens, 4 query / 1 KV head, head dim 64, page 16,
                  identity page table, budget 512 (sink 16, window 64).
* ``llama32k``  - Llama-3.1-8B attention geometry: batch 8, 32 query / 8 KV
                  heads, head dim 128, 32768 tokens each, page 16, budget 2048
                  (sink 64, window 512), 8 needle keys per (sequence, KV head),
                  physical pages a random permutation of a shared pool.
* ``llama128k`` - the same geometry at 131072 tokens per sequence.
* ``ragged``    - batch 4, lengths uniform in [65536, 262144], page 32, budget
                  4096 (sink 128, window 1024), LogNormal(0,1) outlier scales on
                  4 of 128 channels per KV head (applied to K and V).
* ``mla``       - one 576-wide latent per token shared by 128 query heads, value
                  = first 512 latent dims, batch 16 x 65536 tokens, page 64,
                  budget 2048 (sink 64, window 512), values ~ N(0, 0.5^2).
* ``prune``     - 32 sessions, lengths uniform in [8192, 65536], page 16,
                  keep-mask = first 64 + last 2048 tokens + random spans
                  (geometric lengths, mean 256) covering 20% of the middle,
                  then decode with budget 1024 (sink 64, window 512).

Every workload can be shrunk through keyword overrides for tests that must finish fast.
"""

from __future__ import annotations

import dataclasses
import math
import os
from typing import Optional

import numpy as np

__all__ = [
    "Geometry", "DecodeCase", "PruneCase", "WORKLOADS", "f32_to_bf16", "bf16_to_f32",
    "decode_case", "prune_case", "poison_padding", "POISON_BITS",
]

# bf16 bit patterns used to poison storage that must never be read.
POISON_BITS = {
    "nan": 0x7FC1,
    "inf": 0x7F80,
    "ninf": 0xFF80,
    "big": 0x7149,   # ~1e30
}


def f32_to_bf16(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bits, round to nearest even (inputs are finite, so the 32-bit
    sum below cannot overflow: the largest finite pattern is 0xFF7FFFFF)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    r = (u >> 16) & np.uint32(1)
    r += np.uint32(0x7FFF)
    r += u
    r >>= np.uint32(16)
    return r.astype(np.uint16)


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    """bf16 bits -> float32 (exact)."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), int(stream)])))


_CHUNK = 1 << 22


def _normal_bf16(seed: int, stream: int, shape, sigma: float = 1.0) -> np.ndarray:
    """N(0, sigma^2) samples rounded to bf16.  Block c of 2^22 values comes from its own
    stream SeedSequence([seed, stream, c]); blocks are drawn on host threads (numpy
    releases the GIL while filling), the result does not depend on the thread count."""
    from concurrent.futures import ThreadPoolExecutor
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)

    def block(c: int) -> None:
        s0 = c * _CHUNK
        e = min(n, s0 + _CHUNK)
        rng = np.random.Generator(np.random.PCG64(
            np.random.SeedSequence([int(seed), int(stream), c])))
        x = rng.standard_normal(e - s0, dtype=np.float32)
        if sigma != 1.0:
            x *= np.float32(sigma)
        out[s0:e] = f32_to_bf16(x)

    n_blocks = (n + _CHUNK - 1) // _CHUNK
    workers = max(1, min(16, os.cpu_count() or 1, n_blocks))
    if workers == 1:
        for c in range(n_blocks):
            block(c)
    else:
        with ThreadPoolExecutor(max_workers=workers) as ex:
            list(ex.map(block, range(n_blocks)))
    return out.reshape(shape)


@dataclasses.dataclass
class Geometry:
    """Shapes of one paged decode problem (mirrors the C-ABI ``sa_geom``)."""
    B: int
    Hq: int
    Hkv: int
    Dk: int
    Dv: int
    P: int
    max_pages: int
    n_pool: int
    v_aliases_k: int = 0

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv


@dataclasses.dataclass
class DecodeCase:
    """Inputs of one sparse-decode layer call.

    Layouts (bf16 as uint16 bits):
      q          [B, Hq, Dk]
      k_cache    [n_pool, Hkv, P, Dk]   head-major inside a page
      v_cache    [n_pool, Hkv, P, Dv]   (None when V aliases the first Dv dims of K)
      page_table [B, max_pages] int32   logical page -> physical page, -1 unused
      seq_lens   [B] int32              valid tokens per sequence
    budget / sink / window are token counts, multiples of P.
    """
    name: str
    geom: Geometry
    q: np.ndarray
    k_cache: np.ndarray
    v_cache: Optional[np.ndarray]
    page_table: np.ndarray
    seq_lens: np.ndarray
    budget: int
    sink: int
    window: int
    scale: float
    seed: int


@dataclasses.dataclass
class PruneCase:
    """A decode case plus a keep-mask and a list of free pool pages.

    keep       [B, max_pages * P] uint8  (1 = keep token t of session b)
    free_pages [n_free] int32            fresh physical pages, disjoint from the
                                         pages the page table references
    """
    decode: DecodeCase
    keep: np.ndarray
    free_pages: np.ndarray


# --------------------------------------------------------------------------------------
# Workload table
# --------------------------------------------------------------------------------------

WORKLOADS = {
    "tiny": dict(B=1, Hq=4, Hkv=1, Dk=64, Dv=64, P=16, L=(4096, 4096), budget=512,
                 sink=16, window=64, seed=1, identity=True, needles=0, outliers=0,
                 sigma=1.0, mla=False),
    "llama32k": dict(B=8, Hq=32, Hkv=8, Dk=128, Dv=128, P=16, L=(32768, 32768),
                     budget=2048, sink=64, window=512, seed=2, identity=False,
                     needles=8, outliers=0, sigma=1.0, mla=False),
    "llama128k": dict(B=8, Hq=32, Hkv=8, Dk=128, Dv=128, P=16, L=(131072, 131072),
                      budget=2048, sink=64, window=512, seed=22, identity=False,
                      needles=8, outliers=0, sigma=1.0, mla=False),
    "ragged": dict(B=4, Hq=32, Hkv=8, Dk=128, Dv=128, P=32, L=(65536, 262144),
                   budget=4096, sink=128, window=1024, seed=3, identity=False,
                   needles=0, outliers=4, sigma=1.0, mla=False),
    "mla": dict(B=16, Hq=128, Hkv=1, Dk=576, Dv=512, P=64, L=(65536, 65536),
                budget=2048, sink=64, window=512, seed=4, identity=False,
                needles=0, outliers=0, sigma=0.5, mla=True),
    "prune": dict(B=32, Hq=32, Hkv=8, Dk=128, Dv=128, P=16, L=(8192, 65536),
                  budget=1024, sink=64, window=512, seed=5, identity=False,
                  needles=0, outliers=0, sigma=1.0, mla=False),
}

# tensor stream ids (one independent random stream per tensor)
_S_LENS, _S_PERM, _S_Q, _S_K, _S_V, _S_NEEDLE, _S_OUTLIER, _S_KEEP = range(8)


def decode_case(workload: str, *, seed: Optional[int] = None, B: Optional[int] = None,
                L: Optional[tuple] = None, budget: Optional[int] = None,
                sink: Optional[int] = None, window: Optional[int] = None,
                P: Optional[int] = None, Hq: Optional[int] = None, Hkv: Optional[int] = None,
                Dk: Optional[int] = None, identity: Optional[bool] = None,
                needles: Optional[int] = None, seq_lens: Optional[list] = None,
                extra_pool_pages: int = 0, poison: Optional[str] = None,
                scale: Optional[float] = None) -> DecodeCase:
    """Build one seeded decode case; keyword overrides shrink or reshape it for tests.

    ``seq_lens`` (explicit list) overrides the length distribution.  The pool holds
    exactly the referenced pages plus ``extra_pool_pages`` never-referenced ones.
    ``poison`` fills never-valid storage (padding slots of partial pages and
    unreferenced pool pages) with the named bf16 pattern so that any read of
    it shows up as a mismatch.
    """
    w = dict(WORKLOADS[workload])
    for k_, v_ in dict(seed=seed, B=B, L=L, budget=budget, sink=sink, window=window, P=P,
                       Hq=Hq, Hkv=Hkv, Dk=Dk, identity=identity, needles=needles).items():
        if v_ is not None:
            w[k_] = v_
    if Dk is not None and not w["mla"]:
        w["Dv"] = Dk
    seed_ = int(w["seed"])
    Bn, Pn = int(w["B"]), int(w["P"])
    Hq_, Hkv_, Dk_, Dv_ = int(w["Hq"]), int(w["Hkv"]), int(w["Dk"]), int(w["Dv"])

    if seq_lens is not None:
        lens = np.asarray(seq_lens, dtype=np.int32)
        assert lens.shape == (Bn,)
    else:
        lo, hi = w["L"]
        if lo == hi:
            lens = np.full(Bn, lo, dtype=np.int32)
        else:
            lens = _rng(seed_, _S_LENS).integers(lo, hi + 1, size=Bn).astype(np.int32)
    n_pages = (lens.astype(np.int64) + Pn - 1) // Pn
    max_pages = int(max(1, n_pages.max()))
    n_used = int(n_pages.sum())
    n_pool = n_used + int(extra_pool_pages)

    # physical placement: identity (sequence-major) or a random permutation of the pool
    if w["identity"]:
        phys = np.arange(n_used, dtype=np.int64)
    else:
        phys = _rng(seed_, _S_PERM).permutation(n_pool)[:n_used].astype(np.int64)
    page_table = np.full((Bn, max_pages), -1, dtype=np.int32)
    o = 0
    for b in range(Bn):
        nb = int(n_pages[b])
        page_table[b, :nb] = phys[o:o + nb]
        o += nb

    q = _normal_bf16(seed_, _S_Q, (Bn, Hq_, Dk_))
    k_cache = _normal_bf16(seed_, _S_K, (n_pool, Hkv_, Pn, Dk_), w["sigma"])
    v_cache = None if w["mla"] else _normal_bf16(seed_, _S_V, (n_pool, Hkv_, Pn, Dv_),
                                                 w["sigma"])

    if w["outliers"]:
        # per KV head: `outliers` channels scaled by LogNormal(0,1), applied to K and V
        rng = _rng(seed_, _S_OUTLIER)
        for h in range(Hkv_):
            ch = rng.choice(Dk_, size=int(w["outliers"]), replace=False)
            sc = rng.lognormal(0.0, 1.0, size=int(w["outliers"])).astype(np.float32)
            for c, s in zip(ch, sc):
                kk = bf16_to_f32(k_cache[:, h, :, c]) * s
                k_cache[:, h, :, c] = f32_to_bf16(kk)
                if v_cache is not None and c < Dv_:
                    vv = bf16_to_f32(v_cache[:, h, :, c]) * s
                    v_cache[:, h, :, c] = f32_to_bf16(vv)

    if w["needles"]:
        # per (sequence, KV head): keys set to 4 * (unit mean direction of that head's
        # query group) at distinct random token slots of non-forced pages
        rng = _rng(seed_, _S_NEEDLE)
        G = Hq_ // Hkv_
        s_pages, w_pages = int(w["sink"]) // Pn, int(w["window"]) // Pn
        qf = bf16_to_f32(q).astype(np.float64)
        for b in range(Bn):
            nb = int(n_pages[b])
            lo_p, hi_p = s_pages, nb - w_pages      # candidate (non-forced) pages
            if hi_p <= lo_p:
                continue
            for h in range(Hkv_):
                d = qf[b, h * G:(h + 1) * G].mean(axis=0)
                d = 4.0 * d / max(np.linalg.norm(d), 1e-30)
                nd = f32_to_bf16(d.astype(np.float32))
                slots = rng.choice((hi_p - lo_p) * Pn, size=min(int(w["needles"]),
                                                              (hi_p - lo_p) * Pn), replace=False)
                for s in slots:
                    lp = lo_p + int(s) // Pn
                    t = int(s) % Pn
                    if lp * Pn + t >= int(lens[b]):
                        continue
                    k_cache[page_table[b, lp], h, t, :] = nd

    if poison is not None:
        poison_padding(k_cache, v_cache, page_table, lens, Pn, POISON_BITS[poison])

    if w["mla"]:
        geom = Geometry(Bn, Hq_, 1, Dk_, Dv_, Pn, max_pages, n_pool, 1)
    else:
        geom = Geometry(Bn, Hq_, Hkv_, Dk_, Dv_, Pn, max_pages, n_pool, 0)
    sc = float(scale) if scale is not None else 1.0 / math.sqrt(Dk_)
    return DecodeCase(workload, geom, q, k_cache, v_cache, page_table, lens,
                      int(w["budget"]), int(w["sink"]), int(w["window"]), sc, seed_)


def poison_padding(k_cache, v_cache, page_table, seq_lens, P, bits):
    """Fill padding slots of partial pages and unreferenced pool pages with ``bits``."""
    used = np.zeros(k_cache.shape[0], dtype=bool)
    for b in range(page_table.shape[0]):
        L = int(seq_lens[b])
        nb = (L + P - 1) // P
        used[page_table[b, :nb]] = True
        if L % P and nb > 0:
            last = page_table[b, nb - 1]
            k_cache[last, :, L % P:, :] = bits
            if v_cache is not None:
                v_cache[last, :, L % P:, :] = bits
    k_cache[~used] = bits
    if v_cache is not None:
        v_cache[~used] = bits


def keep_mask(lens: np.ndarray, width: int, seed: int, head: int = 64, tail: int = 2048,
              frac: float = 0.2, mean_span: float = 256.0) -> np.ndarray:
    """keep[b, t] = 1 for the first ``head`` and last ``tail`` tokens, plus random spans
    (start uniform in the middle, length ~ Geometric(1/mean_span), clipped) OR-ed in
    until at least ``frac`` of the middle [head, L - tail) is kept."""
    rng = _rng(seed, _S_KEEP)
    B = len(lens)
    keep = np.zeros((B, width), dtype=np.uint8)
    for b in range(B):
        L = int(lens[b])
        keep[b, :min(head, L)] = 1
        keep[b, max(0, L - tail):L] = 1
        lo, hi = head, L - tail
        if hi <= lo:
            continue
        mid = keep[b, lo:hi]
        target = int(math.ceil(frac * (hi - lo)))
        kept = 0
        while kept < target:
            s = int(rng.integers(0, hi - lo))
            ln = int(rng.geometric(1.0 / mean_span))
            e = min(hi - lo, s + ln)
            kept += int((mid[s:e] == 0).sum())
            mid[s:e] = 1
    return keep


def prune_case(workload: str = "prune", *, extra_free: int = 0, keep_all: bool = False,
               keep_none: bool = False, keep_override: Optional[np.ndarray] = None,
               **kw) -> PruneCase:
    """A decode case, its keep-mask and enough fresh pages to compact into.

    The pool is sized for the current pages plus the fresh ones; the fresh pages
    (``free_pages``) are the pool pages no page table references, in a seeded
    random order.
    """
    base = decode_case(workload, **kw)
    g = base.geom
    P = g.P
    width = g.max_pages * P
    if keep_override is not None:
        keep = np.ascontiguousarray(keep_override, dtype=np.uint8)
    elif keep_all:
        keep = np.ones((g.B, width), dtype=np.uint8)
    elif keep_none:
        keep = np.zeros((g.B, width), dtype=np.uint8)
    else:
        keep = keep_mask(base.seq_lens, width, base.seed)
    # valid-range kept counts give the fresh pages needed
    need = 0
    for b in range(g.B):
        L = int(base.seq_lens[b])
        need += (int(keep[b, :L].sum()) + P - 1) // P
    n_free = need + int(extra_free)
    # grow the pool by n_free fresh pages (filled with seeded noise)
    k_new = _normal_bf16(base.seed, 100, (n_free,) + base.k_cache.shape[1:])
    k_cache = np.concatenate([base.k_cache, k_new], axis=0)
    v_cache = None
    if base.v_cache is not None:
        v_new = _normal_bf16(base.seed, 101, (n_free,) + base.v_cache.shape[1:])
        v_cache = np.concatenate([base.v_cache, v_new], axis=0)
    free_pages = (g.n_pool + _rng(base.seed, 102).permutation(n_free)).astype(np.int32)
    geom = dataclasses.replace(g, n_pool=g.n_pool + n_free)
    dec = dataclasses.replace(base, geom=geom, k_cache=k_cache, v_cache=v_cache)
    return PruneCase(dec, keep, free_pages)
