"""sa_sparse_decode across head layouts, page sizes and consecutive calls, against the
oracle and against the library's own selection entry point.

- every supported head layout (1, 2, 4, 8 and 16 KV heads; 1 to 8 query heads per KV
  head), head dims 64 and 128, pages of 16, 32 and 64 tokens, ragged and empty sequences;
- the selection of sa_sparse_decode is bit-identical to sa_select_pages, and both are
  bit-exact with the oracle outside the tie band;
- attention within the stated tolerance of the oracle over that selection;
- many calls in a row on one workspace with changing lengths, budgets and inputs, so that
  scratch left by an earlier call can never leak into a later one;
- bitwise determinism of repeated calls.
"""

import numpy as np
import pytest

import oracle
import synth
from parity import DevCase, check_attention, check_selection, u16

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import paged_kv_cache_sa_b200 as sa  # noqa: E402

CASES = [
    # (workload, overrides)
    ("tiny", dict(B=1, seq_lens=[4096])),
    ("tiny", dict(B=4, seq_lens=[4096, 1, 0, 2500], Hkv=2, Hq=16, poison="nan")),
    ("tiny", dict(B=3, seq_lens=[3000, 17, 5000], Hkv=4, Hq=4, P=32, budget=1024, sink=64,
                  window=128, poison="inf")),
    ("tiny", dict(B=2, seq_lens=[9000, 4200], Hkv=1, Hq=8, P=64, budget=1024, sink=64,
                  window=256, poison="big")),
    ("llama32k", dict(B=3, seq_lens=[8192, 5000, 100], seed=31, poison="nan")),
    ("llama32k", dict(B=2, seq_lens=[6000, 7777], seed=32, Hkv=16, Hq=32)),
    ("llama32k", dict(B=2, seq_lens=[6000, 7777], seed=33, Hkv=4, Hq=32, P=32, budget=1024,
                      sink=64, window=256)),
    ("llama32k", dict(B=2, seq_lens=[6000, 4097], seed=34, Hkv=8, Hq=8, P=64, budget=1024,
                      sink=64, window=0)),
    ("llama32k", dict(B=2, seq_lens=[7000, 3000], seed=35, Dk=64, budget=512, sink=0,
                      window=256)),
    ("ragged", dict(B=2, L=(20000, 30000), seed=36, budget=2048, sink=128, window=512,
                    poison="nan")),
]


def _ids(c):
    wl, kw = c
    return wl + "-" + "-".join("%s%s" % (k, v if not isinstance(v, list) else len(v))
                               for k, v in kw.items())


def _decode(dc, case, ws, budget=None, sink=None, window=None):
    g = dc.g
    budget = case.budget if budget is None else budget
    sink = case.sink if sink is None else sink
    window = case.window if window is None else window
    K = budget // g.P
    sel = torch.full((g.B, g.Hkv, K), 77, dtype=torch.int32, device="cuda")
    cnt = torch.full((g.B, g.Hkv), 77, dtype=torch.int32, device="cuda")
    out, lse = sa.sparse_decode(g, dc.q, dc.k, dc.v, dc.summ, dc.pt, dc.sl, budget, sink, window,
                                case.scale, ws, sel_out=sel, sel_count_out=cnt)
    assert ws.status() == sa.SA_OK
    return sel.cpu().numpy(), cnt.cpu().numpy(), out.cpu().numpy(), lse.cpu().numpy()


def _check(case, dc, res, budget=None, sink=None, window=None):
    budget = case.budget if budget is None else budget
    sink = case.sink if sink is None else sink
    window = case.window if window is None else window
    g = case.geom
    sel, cnt, out, lse = res
    summ = oracle.page_summaries(g, case.k_cache, case.page_table, case.seq_lens)
    sc = oracle.page_scores(g, case.q, summ, case.page_table, case.seq_lens)
    osel, ocnt = oracle.select_pages(g, sc, case.seq_lens, budget, sink, window)
    tied = check_selection(g, case.seq_lens, budget, sink, window, sc, osel, ocnt, sel, cnt)
    o, l = oracle.attend(g, case.q, case.k_cache, case.v_cache, case.page_table, case.seq_lens,
                         sel if tied else osel, ocnt, case.scale)
    check_attention(out, lse, o, l)


@pytest.mark.parametrize("c", CASES, ids=_ids)
def test_decode_matches_oracle_and_select_pages(c):
    wl, kw = c
    case = synth.decode_case(wl, **kw)
    dc = DevCase(case)
    g = dc.g
    sa.page_summaries(g, dc.k, dc.pt, dc.sl, dc.summ)
    ws = sa.Workspace.for_decode(g, case.budget)
    res = _decode(dc, case, ws)
    _check(case, dc, res)
    # the selection entry point chooses exactly the same pages
    sel_s, cnt_s = sa.select_pages(g, dc.q, dc.summ, dc.pt, dc.sl, case.budget, case.sink,
                                   case.window, ws)
    assert ws.status() == sa.SA_OK
    assert np.array_equal(sel_s.cpu().numpy(), res[0])
    assert np.array_equal(cnt_s.cpu().numpy(), res[1])
    # and a second call on the same workspace is bitwise the same
    res2 = _decode(dc, case, ws)
    for a, b in zip(res, res2):
        assert np.array_equal(a, b)


def test_decode_consecutive_calls_with_changing_inputs():
    # one workspace sized for the largest call; lengths, budgets, queries and the number
    # of pages change from call to call, so an earlier call's scratch sits where a later
    # call reads
    big = synth.decode_case("llama32k", B=3, seq_lens=[12000, 9000, 7000], seed=41)
    g = sa.Geometry.of(big.geom)
    ws = sa.Workspace.for_decode(g, 2048)
    plans = [
        (dict(seq_lens=[12000, 9000, 7000], seed=41), 2048, 64, 512),
        (dict(seq_lens=[3000, 9000, 0], seed=42), 1024, 64, 256),
        (dict(seq_lens=[12000, 1, 6000], seed=43), 2048, 0, 512),
        (dict(seq_lens=[5000, 5000, 5000], seed=44), 512, 16, 64),
        (dict(seq_lens=[12000, 9000, 7000], seed=41), 2048, 64, 512),
    ]
    results = []
    for kw, budget, sink, window in plans:
        case = synth.decode_case("llama32k", B=3, budget=budget, sink=sink, window=window,
                                 **kw)
        dc = DevCase(case)
        # every call here needs at most the first call's workspace
        assert sa.decode_workspace_size(dc.g, budget) <= ws.nbytes
        sa.page_summaries(dc.g, dc.k, dc.pt, dc.sl, dc.summ)
        res = _decode(dc, case, ws)
        _check(case, dc, res)
        results.append(res)
    for a, b in zip(results[0], results[-1]):  # the same inputs again: the same bits
        assert np.array_equal(a, b)


def test_decode_newest_page_refresh():
    # the newest page's summary is stale (as after an append): the call recomputes it from
    # K before choosing, exactly as sa_update_summaries would
    case = synth.decode_case("llama32k", B=2, seq_lens=[9001, 6000], seed=45)
    dc = DevCase(case)
    g = dc.g
    sa.page_summaries(g, dc.k, dc.pt, dc.sl, dc.summ)
    summ_ok = u16(dc.summ).copy()
    P = g.P
    for b, L in enumerate(case.seq_lens):
        last = case.page_table[b, (int(L) + P - 1) // P - 1]
        dc.summ[last] = 0  # a stale summary of the newest page
    ws = sa.Workspace.for_decode(g, case.budget)
    K = case.budget // P
    sel = torch.empty((g.B, g.Hkv, K), dtype=torch.int32, device="cuda")
    cnt = torch.empty((g.B, g.Hkv), dtype=torch.int32, device="cuda")
    out, lse = sa.sparse_decode(g, dc.q, dc.k, dc.v, dc.summ, dc.pt, dc.sl, case.budget,
                                case.sink, case.window, case.scale, ws, sel_out=sel,
                                sel_count_out=cnt, n_tail_refresh=1)
    assert ws.status() == sa.SA_OK
    assert np.array_equal(u16(dc.summ), summ_ok)
    _check(case, dc, (sel.cpu().numpy(), cnt.cpu().numpy(), out.cpu().numpy(),
                      lse.cpu().numpy()))
