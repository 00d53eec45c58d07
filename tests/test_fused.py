"""sa_sparse_decode_fused: the whole decode step in one persistent launch.

The same selection, bit for bit, and the same attention outputs, bit for bit, as
sa_sparse_decode on the same inputs (the phases run the same CTA programs, with the same
work split), and both within the stated tolerance of the oracle.  Covers head layouts,
page sizes, ragged and empty sequences, poisoned padding, the newest-page refresh, and
the Llama-geometry bench size.
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

CASES = {
    "tiny_gqa4": dict(wl="tiny", B=3, seq_lens=[4096, 700, 0], Hkv=2, Hq=8, poison="nan"),
    "tiny_p32_d128": dict(wl="tiny", B=2, seq_lens=[6000, 2500], Hkv=4, Hq=16, Dk=128, P=32,
                          budget=1024, sink=64, window=128, poison="inf"),
    "tiny_p64": dict(wl="tiny", B=2, seq_lens=[9000, 64], Hkv=2, Hq=16, P=64, budget=1024,
                     sink=64, window=128),
    "llama_small": dict(wl="llama32k", B=2, L=(8192, 8192), seed=91),
    "ragged_small": dict(wl="ragged", B=2, seq_lens=[20000, 9000], seed=92),
    "llama32k": dict(wl="llama32k"),
}


@pytest.mark.parametrize("name", list(CASES))
def test_fused_matches_separate_kernels_and_oracle(name):
    kw = dict(CASES[name])
    case = synth.decode_case(kw.pop("wl"), **kw)
    dc = DevCase(case)
    g = dc.g
    K = case.budget // g.P
    sa.page_summaries(g, dc.k, dc.pt, dc.sl, dc.summ)
    # every call refreshes the newest pages' summaries: the same values again
    summ_ref = oracle.page_summaries(case.geom, case.k_cache, case.page_table, case.seq_lens)
    ws = sa.Workspace.for_decode(g, case.budget)
    runs = []
    for fn in (sa.sparse_decode, sa.sparse_decode_fused, sa.sparse_decode_fused):
        sel = torch.full((g.B, g.Hkv, K), 7, dtype=torch.int32, device="cuda")
        cnt = torch.full((g.B, g.Hkv), 7, dtype=torch.int32, device="cuda")
        out, lse = fn(g, dc.q, dc.k, dc.v, dc.summ, dc.pt, dc.sl, case.budget, case.sink,
                      case.window, case.scale, ws, sel_out=sel, sel_count_out=cnt,
                      n_tail_refresh=1)
        assert ws.status() == sa.SA_OK
        assert np.array_equal(u16(dc.summ), summ_ref)
        runs.append((sel.cpu().numpy(), cnt.cpu().numpy(), out.cpu().numpy(),
                     lse.cpu().numpy()))
    for r in runs[1:]:
        for x, y in zip(r, runs[0]):
            assert np.array_equal(x, y)
    # against the oracle
    sc = oracle.page_scores(case.geom, case.q, summ_ref, case.page_table, case.seq_lens)
    osel, ocnt = oracle.select_pages(case.geom, sc, case.seq_lens, case.budget, case.sink,
                                     case.window)
    gs, gc, out, lse = runs[1]
    tied = check_selection(case.geom, case.seq_lens, case.budget, case.sink, case.window, sc,
                           osel, ocnt, gs, gc)
    o, l = oracle.attend(case.geom, case.q, case.k_cache, case.v_cache, case.page_table,
                         case.seq_lens, gs if tied else osel, ocnt, case.scale)
    check_attention(out, lse, o, l)


def test_fused_refuses_the_latent_geometry():
    g = sa.Geometry(B=1, Hq=128, Hkv=1, Dk=576, Dv=512, P=64, max_pages=16, n_pool=16,
                    v_aliases_k=1)
    ws = sa.Workspace.for_decode(g, 512)
    q = torch.zeros((1, 128, 576), dtype=torch.int16, device="cuda")
    kv = torch.zeros((16, 1, 64, 576), dtype=torch.int16, device="cuda")
    summ = torch.zeros((16, 1, 2, 576), dtype=torch.int16, device="cuda")
    pt = torch.zeros((1, 16), dtype=torch.int32, device="cuda")
    sl = torch.zeros((1,), dtype=torch.int32, device="cuda")
    with pytest.raises(sa.SaError) as e:
        sa.sparse_decode_fused(g, q, kv, kv, summ, pt, sl, 512, 64, 128, 0.04, ws)
    assert e.value.status == sa.SA_ERR_UNSUPPORTED
