"""Shared helpers of the GPU parity tests: move a seeded case to the device, run the
library's C ABI through the binding, and compare with the CPU oracle.

Comparison rules:
  * summaries, selections, compaction outputs: bit-exact;
  * a selection may differ from the oracle's only for a (sequence, KV head) whose
    oracle k-th and (k+1)-th candidate scores differ by less than 1e-5 relative; the
    GPU set must then hold every candidate scoring above the band, none below it, and
    all forced pages, and attention is compared with the oracle run over the GPU's
    own selection;
  * attention: max |out - ref| <= 1e-2 and ||out - ref||_2 / ||ref||_2 <= 5e-3 against
    the fp64 oracle; lse within 1e-3.
"""

import numpy as np
import torch

import oracle

OUT_MAX_ABS = 1e-2
OUT_REL_L2 = 5e-3
LSE_MAX_ABS = 1e-3
TIE_REL = 1e-5


def to_dev(a, dev="cuda"):
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a).to(dev)


def u16(t):
    return t.cpu().numpy().view(np.uint16)


class DevCase:
    """Device copies of a synth.DecodeCase."""

    def __init__(self, case, dev="cuda"):
        import paged_kv_cache_sa_b200 as sa
        self.case = case
        self.g = sa.Geometry.of(case.geom)
        self.q = to_dev(case.q, dev)
        self.k = to_dev(case.k_cache, dev)
        self.v = to_dev(case.v_cache, dev) if case.v_cache is not None else None
        self.pt = to_dev(case.page_table, dev)
        self.sl = to_dev(case.seq_lens, dev)
        self.summ = torch.zeros((self.g.n_pool, self.g.Hkv, 2, self.g.Dk), dtype=torch.int16,
                                device=dev)


def run_decode(dc, budget=None, sink=None, window=None, ws=None, scores=True):
    import paged_kv_cache_sa_b200 as sa
    c = dc.case
    budget = c.budget if budget is None else budget
    sink = c.sink if sink is None else sink
    window = c.window if window is None else window
    g = dc.g
    K = budget // g.P
    if ws is None:
        ws = sa.Workspace.for_decode(g, budget)
    sa.page_summaries(g, dc.k, dc.pt, dc.sl, dc.summ)
    sc = None
    if scores:
        sc = torch.empty((g.B, g.Hkv, g.max_pages), dtype=torch.float32, device=dc.q.device)
        sel_s, cnt_s = sa.select_pages(g, dc.q, dc.summ, dc.pt, dc.sl, budget, sink, window, ws,
                                       scores=sc)
    sel = torch.empty((g.B, g.Hkv, K), dtype=torch.int32, device=dc.q.device)
    cnt = torch.empty((g.B, g.Hkv), dtype=torch.int32, device=dc.q.device)
    out, lse = sa.sparse_decode(g, dc.q, dc.k, dc.v, dc.summ, dc.pt, dc.sl, budget, sink, window,
                                c.scale, ws, sel_out=sel, sel_count_out=cnt)
    st = ws.status()
    assert st == sa.SA_OK, sa.STATUS.get(st)
    res = dict(summ=u16(dc.summ), sel=sel.cpu().numpy(), cnt=cnt.cpu().numpy(),
               out=out.cpu().numpy(), lse=lse.cpu().numpy())
    if scores:
        res["scores"] = sc.cpu().numpy()
        res["sel_select"] = sel_s.cpu().numpy()
        res["cnt_select"] = cnt_s.cpu().numpy()
    return res


def check_selection(geom, seq_lens, budget, sink, window, o_scores, o_sel, o_cnt, g_sel, g_cnt):
    """Bit-exact selection, except inside the tie band.  Returns the set of (b, h)
    compared under the tie-band rule."""
    P = geom.P
    K, s, w = budget // P, sink // P, window // P
    k_top = K - s - w
    tied = set()
    assert np.array_equal(o_cnt, g_cnt), "selection counts differ"
    for b in range(geom.B):
        nb = (int(seq_lens[b]) + P - 1) // P
        for h in range(geom.Hkv):
            if np.array_equal(o_sel[b, h], g_sel[b, h]):
                continue
            assert nb > K, "all pages must be selected when n_b <= K (b=%d h=%d)" % (b, h)
            cand = np.arange(s, nb - w)
            sc = o_scores[b, h, cand]
            order = np.lexsort((cand, -sc))
            s_k, s_k1 = sc[order[k_top - 1]], sc[order[k_top]]
            assert abs(s_k - s_k1) < TIE_REL * max(abs(s_k), 1e-30), \
                "selection differs outside the tie band (b=%d h=%d, s_k=%r s_k1=%r)" % (
                    b, h, s_k, s_k1)
            d = TIE_REL * abs(s_k)
            gsel = set(g_sel[b, h, :g_cnt[b, h]].tolist())
            assert list(g_sel[b, h, :g_cnt[b, h]]) == sorted(gsel)
            for p, v in zip(cand, sc):
                if v > s_k + d:
                    assert p in gsel
                if v < s_k1 - d:
                    assert p not in gsel
            assert set(range(s)) <= gsel and set(range(nb - w, nb)) <= gsel
            tied.add((b, h))
    return tied


def check_attention(out, lse, ref_out, ref_lse):
    err = float(np.abs(out - ref_out).max()) if out.size else 0.0
    den = float(np.linalg.norm(ref_out))
    rel = float(np.linalg.norm(out - ref_out)) / den if den > 0 else float(np.linalg.norm(out))
    assert err <= OUT_MAX_ABS, "max |out - ref| = %.3e" % err
    assert rel <= OUT_REL_L2, "rel-L2 = %.3e" % rel
    fin = np.isfinite(ref_lse)
    assert np.array_equal(fin, np.isfinite(lse)), "lse finiteness differs"
    lerr = float(np.abs(lse[fin] - ref_lse[fin]).max()) if fin.any() else 0.0
    assert lerr <= LSE_MAX_ABS, "max |lse - ref| = %.3e" % lerr
    return err, rel, lerr


def full_parity(case, res, budget=None, sink=None, window=None):
    """Compare one run_decode() result with the oracle end to end."""
    budget = case.budget if budget is None else budget
    sink = case.sink if sink is None else sink
    window = case.window if window is None else window
    g = case.geom
    summ = oracle.page_summaries(g, case.k_cache, case.page_table, case.seq_lens)
    assert np.array_equal(res["summ"], summ), "summaries differ"
    sc = oracle.page_scores(g, case.q, summ, case.page_table, case.seq_lens)
    if "scores" in res:
        fin = np.isfinite(sc)
        assert np.array_equal(fin, np.isfinite(res["scores"]))
        assert np.allclose(res["scores"][fin], sc[fin], rtol=1e-5, atol=1e-4), \
            "scores differ: %.3e" % np.abs(res["scores"][fin] - sc[fin]).max()
    o_sel, o_cnt = oracle.select_pages(g, sc, case.seq_lens, budget, sink, window)
    tied = check_selection(g, case.seq_lens, budget, sink, window, sc, o_sel, o_cnt, res["sel"],
                           res["cnt"])
    if "sel_select" in res:
        assert np.array_equal(res["sel_select"], res["sel"])
        assert np.array_equal(res["cnt_select"], res["cnt"])
    att_sel = res["sel"] if tied else o_sel
    out, lse = oracle.attend(g, case.q, case.k_cache, case.v_cache, case.page_table,
                             case.seq_lens, att_sel, o_cnt, case.scale)
    return check_attention(res["out"], res["lse"], out, lse) + (len(tied),)
