"""Selection over long sequences (2K to 16K pages per sequence), against the oracle.

Quest, section 3: each (sequence, KV head) keeps its top-K pages by upper bound, the sink
and window pages always; equal scores are taken lowest page first.  At these lengths
the radix passes see thousands of keys per pair, the boundary bin is fuller and the
selection's key loads and list passes are longest.  Covered:

- 2188 to 16384 pages; page sizes 16 and 32; identity and shuffled page tables;
  sequences that fit the budget (no selection), just exceed it, and are long; NaN in the
  padding of partial pages;
- exact ties at 4375 and 8192 pages: all-equal scores (the lowest pages win) and
  small-integer scores (many members in the boundary bin, ranked exactly);
- the same selection, bit for bit, from sa_select_pages, sa_sparse_decode and (where it
  takes the geometry) sa_sparse_decode_fused.
"""

import numpy as np
import pytest

import oracle
import synth
from parity import DevCase, full_parity, run_decode

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import paged_kv_cache_sa_b200 as sa  # noqa: E402


CASES = [
    # 4096 pages
    dict(B=3, seq_lens=[40000, 3000, 65536], Hkv=2, Hq=4, budget=4096, sink=64, window=256,
         seed=201, identity=False),
    # 4375 pages, one sequence within the budget, NaN padding
    dict(B=3, seq_lens=[70000, 4096, 33001], Hkv=2, Hq=8, budget=4096, sink=16, window=512,
         seed=202, poison="nan"),
    # 8192 pages, head dim 128
    dict(B=2, seq_lens=[131072, 40000], Hkv=2, Hq=4, Dk=128, budget=4096, sink=64,
         window=256, seed=203, identity=False),
    # 16384 pages, no sink and no window, a sequence just over the budget
    dict(B=3, seq_lens=[262144, 100, 8209], Hkv=1, Hq=2, budget=8192, sink=0, window=0,
         seed=204),
    # page 32, 2188 pages
    dict(B=2, seq_lens=[70000, 65600], Hkv=2, Hq=4, P=32, budget=2048, sink=32, window=128,
         seed=205, identity=False),
]


def _ids(kw):
    return "pages%d-%s" % (_max_pages(kw), kw["seed"])


def _max_pages(kw):
    P = kw.get("P", 16)
    return -(-max(kw["seq_lens"]) // P)


def _fused_selection(dc, case):
    """The selection of sa_sparse_decode_fused (one CTA per pair), or None when that entry
    point does not take this geometry."""
    g = dc.g
    K = case.budget // g.P
    ws = sa.Workspace.for_decode(g, case.budget)
    sel = torch.empty((g.B, g.Hkv, K), dtype=torch.int32, device="cuda")
    cnt = torch.empty((g.B, g.Hkv), dtype=torch.int32, device="cuda")
    try:
        sa.sparse_decode_fused(g, dc.q, dc.k, dc.v, dc.summ, dc.pt, dc.sl, case.budget,
                               case.sink, case.window, case.scale, ws, sel_out=sel,
                               sel_count_out=cnt)
    except sa.SaError as e:
        if e.status == sa.SA_ERR_UNSUPPORTED:
            return None
        raise
    assert ws.status() == sa.SA_OK
    return sel.cpu().numpy(), cnt.cpu().numpy()


@pytest.mark.parametrize("kw", CASES, ids=_ids)
def test_long_selection_matches_oracle(kw):
    assert _max_pages(kw) > 2048
    case = synth.decode_case("tiny", **kw)
    assert case.geom.max_pages == _max_pages(kw)
    dc = DevCase(case)
    res = run_decode(dc)
    full_parity(case, res)
    # sa_select_pages and sa_sparse_decode: the same selection
    assert np.array_equal(res["sel_select"], res["sel"])
    assert np.array_equal(res["cnt_select"], res["cnt"])
    fused = _fused_selection(dc, case)
    if fused is not None:
        assert np.array_equal(fused[0], res["sel"])
        assert np.array_equal(fused[1], res["cnt"])


@pytest.mark.parametrize("mode", ["zero_q", "quantized"])
@pytest.mark.parametrize("lens", [[70000, 40000], [131072, 2000]], ids=["p4375", "p8192"])
def test_long_selection_exact_ties_lowest_index(mode, lens):
    # Scores with many exact ties around the k-th place, exact on both sides (all zero,
    # or small integer sums): the lowest page indices win, bit-exactly.
    case = synth.decode_case("tiny", B=2, seq_lens=lens, Hkv=2, Hq=4, budget=4096, sink=16,
                             window=64, seed=211)
    assert case.geom.max_pages > 4096
    rng = np.random.default_rng(211)
    if mode == "zero_q":
        case.q[...] = 0
    else:
        vals = np.array([0xBF80, 0x0000, 0x3F80], dtype=np.uint16)          # -1, 0, 1
        case.q[...] = vals[rng.integers(0, 3, size=case.q.shape)]
        kv = np.array([0xC000, 0xBF80, 0x0000, 0x3F80, 0x4000], dtype=np.uint16)  # -2..2
        case.k_cache[...] = kv[rng.integers(0, 5, size=case.k_cache.shape)]
    dc = DevCase(case)
    res = run_decode(dc)
    g = case.geom
    summ = oracle.page_summaries(g, case.k_cache, case.page_table, case.seq_lens)
    sc = oracle.page_scores(g, case.q, summ, case.page_table, case.seq_lens)
    o_sel, o_cnt = oracle.select_pages(g, sc, case.seq_lens, case.budget, case.sink,
                                       case.window)
    assert np.array_equal(res["cnt"], o_cnt)
    assert np.array_equal(res["sel"], o_sel)
    assert np.array_equal(res["sel_select"], o_sel)
    fin = np.isfinite(sc)
    assert np.array_equal(res["scores"][fin], sc[fin].astype(np.float32))
    full_parity(case, res)
    fused = _fused_selection(dc, case)
    if fused is not None:
        assert np.array_equal(fused[0], o_sel)
