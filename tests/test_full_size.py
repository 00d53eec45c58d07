"""Parity at the full benchmark sizes.

bench.py decodes every layer with sa_sparse_decode, whose two halves are sa_select_pages
(newest page's summary refreshed, physical pages of the selection returned) and
sa_attend_selected over those physical pages: the same kernels in the same launch
configuration.  Here the two halves run once on the full workloads and every output is
compared with the oracle:
- summaries bit-exact;
- selection bit-exact outside the tie band;
- attention within the stated tolerance;
and the bench's own sa_sparse_decode call (twice, the second on a reused workspace) gives
bitwise the same outputs as the two halves.

The workloads are:
- Llama-3.1-8B geometry, batch 8, 32/8 heads, head dim 128, at 32K and 128K tokens;
- the ragged long-context batch: 4 sequences of 64K-256K tokens, page 32;
- the latent geometry: 16 x 64K tokens, 128 heads on one 576-wide latent.
"""

import numpy as np
import pytest

import synth
import oracle
from parity import DevCase, check_attention, check_selection, u16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("wl", ["llama32k", "llama128k", "ragged", "mla"])
def test_full_size_bench_launch_config(wl):
    import torch
    import paged_kv_cache_sa_b200 as sa
    case = synth.decode_case(wl)
    dc = DevCase(case)
    g = dc.g
    K = case.budget // g.P
    sa.page_summaries(g, dc.k, dc.pt, dc.sl, dc.summ)
    ws = sa.Workspace.for_decode(g, case.budget)
    sel = torch.empty((g.B, g.Hkv, K), dtype=torch.int32, device="cuda")
    cnt = torch.empty((g.B, g.Hkv), dtype=torch.int32, device="cuda")
    phys = torch.empty_like(sel)
    scores = torch.empty((g.B, g.Hkv, g.max_pages), dtype=torch.float32, device="cuda")
    sa.select_pages(g, dc.q, dc.summ, dc.pt, dc.sl, case.budget, case.sink, case.window, ws,
                    sel=sel, sel_count=cnt, k_cache=dc.k, n_tail_refresh=1, sel_phys=phys,
                    scores=scores)
    out, lse = sa.attend_selected(g, dc.q, dc.k, dc.v, dc.pt, dc.sl, sel, cnt, case.scale, ws,
                                  sel_phys=phys)
    assert ws.status() == sa.SA_OK
    gs, gc = sel.cpu().numpy(), cnt.cpu().numpy()

    summ = oracle.page_summaries(case.geom, case.k_cache, case.page_table, case.seq_lens)
    assert np.array_equal(u16(dc.summ), summ)
    sc = oracle.page_scores(case.geom, case.q, summ, case.page_table, case.seq_lens)
    fin = np.isfinite(sc)
    gsc = scores.cpu().numpy()
    assert np.array_equal(fin, np.isfinite(gsc))
    assert np.allclose(gsc[fin], sc[fin], rtol=1e-5, atol=1e-4)
    osel, ocnt = oracle.select_pages(case.geom, sc, case.seq_lens, case.budget, case.sink,
                                     case.window)
    tied = check_selection(case.geom, case.seq_lens, case.budget, case.sink, case.window, sc,
                           osel, ocnt, gs, gc)
    # the physical pages handed to attention are the page-table entries of the selection
    pt = case.page_table
    gp = phys.cpu().numpy()
    for b in range(g.B):
        for h in range(g.Hkv):
            c = gc[b, h]
            assert np.array_equal(gp[b, h, :c], pt[b, gs[b, h, :c]])
            assert (gp[b, h, c:] == -1).all()
    o, l = oracle.attend(case.geom, case.q, case.k_cache, case.v_cache, case.page_table,
                         case.seq_lens, gs if tied else osel, ocnt, case.scale)
    check_attention(out.cpu().numpy(), lse.cpu().numpy(), o, l)
    # the bench's own call (twice, so the second runs on a reused workspace): the same
    # selection and bitwise the same outputs
    for _ in range(2):
        sel2 = torch.empty_like(sel)
        cnt2 = torch.empty_like(cnt)
        out2, lse2 = sa.sparse_decode(g, dc.q, dc.k, dc.v, dc.summ, dc.pt, dc.sl, case.budget,
                                      case.sink, case.window, case.scale, ws, sel_out=sel2,
                                      sel_count_out=cnt2, n_tail_refresh=1)
        assert ws.status() == sa.SA_OK
        assert np.array_equal(sel2.cpu().numpy(), gs)
        assert np.array_equal(cnt2.cpu().numpy(), gc)
        assert np.array_equal(u16(dc.summ), summ)
        assert np.array_equal(out2.cpu().numpy(), out.cpu().numpy())
        assert np.array_equal(lse2.cpu().numpy(), lse.cpu().numpy())


def test_prune_full_size_bench_config():
    """Prefix-cache pruning compaction at the size bench.py times (SparseEngine blog,
    Prefix-Cache Pruning paragraph): 32 sessions of 8K-64K tokens, page 16, 8 KV heads,
    keep-mask of sink + window + random spans.  Every output bit-exact: new page table,
    lengths, position map, logical lengths, the whole K/V pool and the new pages'
    summaries."""
    import torch
    import paged_kv_cache_sa_b200 as sa
    pc = synth.prune_case("prune")
    d = pc.decode
    g = sa.Geometry.of(d.geom)
    assert g.B == 32
    to_dev = lambda a: torch.from_numpy(np.ascontiguousarray(
        a.view(np.int16) if a.dtype == np.uint16 else a)).cuda()
    k, v = to_dev(d.k_cache), to_dev(d.v_cache)
    summ = torch.zeros((g.n_pool, g.Hkv, 2, g.Dk), dtype=torch.int16, device="cuda")
    ws = sa.Workspace.for_prune(g)
    npt, nsl, pos, ll = sa.prune_compact(g, k, v, to_dev(d.page_table), to_dev(d.seq_lens),
                                         to_dev(pc.keep), to_dev(pc.free_pages), k, v, summ, ws)
    assert ws.status() == sa.SA_OK
    ref = oracle.prune_compact(d.geom, d.k_cache, d.v_cache, d.page_table, d.seq_lens, pc.keep,
                               pc.free_pages)
    assert np.array_equal(npt.cpu().numpy(), ref["new_page_table"])
    assert np.array_equal(nsl.cpu().numpy(), ref["new_seq_lens"])
    assert np.array_equal(pos.cpu().numpy(), ref["pos_map"])
    assert np.array_equal(ll.cpu().numpy(), ref["logical_len"])
    assert np.array_equal(u16(k), ref["k_dst"])
    assert np.array_equal(u16(v), ref["v_dst"])
    assert np.array_equal(u16(summ), ref["summ"])
