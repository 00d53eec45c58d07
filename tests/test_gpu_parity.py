"""GPU parity of every C-ABI entry point against the CPU oracle (needs a B200)."""

import dataclasses

import numpy as np
import pytest

import oracle
import synth
from parity import (DevCase, check_attention, check_selection, full_parity, run_decode, to_dev,
                    u16)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import paged_kv_cache_sa_b200 as sa  # noqa: E402


# ------------------------------------------------------------------------------------
# summaries (bit-exact)
# ------------------------------------------------------------------------------------

@pytest.mark.parametrize("wl,P,Dk,lens", [
    ("tiny", 16, 64, [0, 1, 15, 16, 17, 4096]),
    ("tiny", 32, 128, [31, 32, 33, 1000]),
    ("tiny", 64, 128, [1, 63, 64, 65, 700]),
    ("mla", 64, None, [1, 65, 640]),
])
def test_summaries_bit_exact(wl, P, Dk, lens):
    kw = dict(B=len(lens), seq_lens=lens, P=P, identity=False, extra_pool_pages=4, poison="nan")
    if wl == "tiny":
        kw.update(Dk=Dk, Hkv=4, Hq=8)
    else:
        kw.update(Hq=128, budget=640, sink=64, window=128)
    case = synth.decode_case(wl, **kw)
    dc = DevCase(case)
    sa.page_summaries(dc.g, dc.k, dc.pt, dc.sl, dc.summ)
    ref = oracle.page_summaries(case.geom, case.k_cache, case.page_table, case.seq_lens)
    assert np.array_equal(u16(dc.summ), ref)


def test_signed_zero_summaries():
    case = synth.decode_case("tiny", B=1, seq_lens=[40], Hkv=1, Hq=4)
    k = case.k_cache.copy()
    k[:, :, :, 0] = 0x8000
    k[:, :, 1::2, 0] = 0x0000     # -0 and +0 alternate in channel 0
    k[:, :, :, 1] = 0x0000
    case = dataclasses.replace(case, k_cache=k)
    dc = DevCase(case)
    sa.page_summaries(dc.g, dc.k, dc.pt, dc.sl, dc.summ)
    ref = oracle.page_summaries(case.geom, case.k_cache, case.page_table, case.seq_lens)
    assert np.array_equal(u16(dc.summ), ref)


def test_update_summaries_tail_pages():
    # the pool already holds one appended token per sequence; summaries were computed
    # before the append, so only each sequence's last page is stale
    case = synth.decode_case("tiny", B=3, seq_lens=[1001, 17, 4097], Hkv=2, Hq=8,
                             poison="nan")
    dc = DevCase(case)
    before = to_dev(case.seq_lens - 1)
    sa.page_summaries(dc.g, dc.k, dc.pt, before, dc.summ)
    sa.update_summaries(dc.g, dc.k, dc.pt, dc.sl, dc.summ, n_tail_pages=1)
    ref = oracle.page_summaries(case.geom, case.k_cache, case.page_table, case.seq_lens)
    assert np.array_equal(u16(dc.summ), ref)


def test_fused_tail_refresh_in_selection():
    # stale summaries for the newest page; select_pages refreshes them from K first
    case = synth.decode_case("llama32k", B=3, seq_lens=[4097, 3000, 2064], seed=41,
                             poison="nan")
    dc = DevCase(case)
    before = to_dev(np.maximum(case.seq_lens - 1, 0))
    sa.page_summaries(dc.g, dc.k, dc.pt, before, dc.summ)
    ws = sa.Workspace.for_decode(dc.g, case.budget)
    sel, cnt = sa.select_pages(dc.g, dc.q, dc.summ, dc.pt, dc.sl, case.budget, case.sink,
                               case.window, ws, k_cache=dc.k, n_tail_refresh=1)
    assert ws.status() == sa.SA_OK
    ref = oracle.page_summaries(case.geom, case.k_cache, case.page_table, case.seq_lens)
    assert np.array_equal(u16(dc.summ), ref)
    sc = oracle.page_scores(case.geom, case.q, ref, case.page_table, case.seq_lens)
    osel, ocnt = oracle.select_pages(case.geom, sc, case.seq_lens, case.budget, case.sink,
                                     case.window)
    from parity import check_selection
    check_selection(case.geom, case.seq_lens, case.budget, case.sink, case.window, sc, osel,
                    ocnt, sel.cpu().numpy(), cnt.cpu().numpy())


def test_workspace_reuse_across_calls():
    # counters inside a workspace return to zero after every call: many calls in a row
    # on the same workspace (and interleaved with another geometry's workspace) stay exact
    c1 = synth.decode_case("llama32k", B=2, L=(4096, 4096), seed=51)
    c2 = synth.decode_case("llama32k", B=2, seq_lens=[1000, 4000], seed=52)
    d1, d2 = DevCase(c1), DevCase(c2)
    w1 = sa.Workspace.for_decode(d1.g, c1.budget)
    w2 = sa.Workspace.for_decode(d2.g, c2.budget)
    for _ in range(3):
        full_parity(c1, run_decode(d1, ws=w1))
        full_parity(c2, run_decode(d2, ws=w2))


# ------------------------------------------------------------------------------------
# scoring + selection + attention, small end-to-end cases
# ------------------------------------------------------------------------------------

SMALL = [
    dict(wl="tiny"),
    dict(wl="tiny", B=3, seq_lens=[4096, 700, 50], Hkv=2, Hq=8, poison="nan"),
    dict(wl="tiny", B=2, seq_lens=[0, 1], Hkv=1, Hq=4),
    dict(wl="tiny", B=2, seq_lens=[513, 511], Hkv=1, Hq=4, budget=512, sink=0, window=0),
    dict(wl="tiny", B=1, seq_lens=[3000], Hkv=1, Hq=1, budget=1024, sink=16, window=1008),
    dict(wl="tiny", B=2, seq_lens=[5000, 2049], Hkv=2, Hq=16, P=32, budget=1024, sink=32,
         window=256, poison="inf"),
    dict(wl="tiny", B=2, seq_lens=[9000, 3333], Hkv=1, Hq=6, P=64, budget=1024, sink=64,
         window=256, poison="big"),
    dict(wl="llama32k", B=2, L=(8192, 8192), seed=12, poison="nan"),
    dict(wl="llama32k", B=2, L=(4096, 4096), seed=13, P=32, budget=1024, sink=64, window=256),
    dict(wl="llama32k", B=2, L=(4096, 4096), seed=14, P=64, budget=1024, sink=64, window=256),
    dict(wl="ragged", B=2, L=(3000, 9000), seed=15, budget=1024, sink=128, window=256,
         poison="nan"),
]


@pytest.mark.parametrize("kw", SMALL, ids=lambda kw: "-".join(
    "%s%s" % (k, v if not isinstance(v, list) else len(v)) for k, v in kw.items()))
def test_decode_parity_small(kw):
    kw = dict(kw)
    wl = kw.pop("wl")
    case = synth.decode_case(wl, **kw)
    res = run_decode(DevCase(case))
    full_parity(case, res)


@pytest.mark.parametrize("mode", ["zero_q", "quantized"])
def test_selection_exact_ties_lowest_index(mode):
    # Scores with many exact ties around the k-th place, computed exactly on both sides
    # (all zero, or small integer sums): the lowest page indices must win, bit-exactly.
    case = synth.decode_case("tiny", B=2, seq_lens=[4096, 3000], Hkv=2, Hq=8, budget=512,
                             sink=16, window=64, seed=61)
    rng = np.random.default_rng(61)
    if mode == "zero_q":
        case.q[...] = 0
    else:
        vals = np.array([0xBF80, 0x0000, 0x3F80], dtype=np.uint16)          # -1, 0, 1
        case.q[...] = vals[rng.integers(0, 3, size=case.q.shape)]
        kv = np.array([0xC000, 0xBF80, 0x0000, 0x3F80, 0x4000], dtype=np.uint16)  # -2..2
        case.k_cache[...] = kv[rng.integers(0, 5, size=case.k_cache.shape)]
    res = run_decode(DevCase(case))
    g = case.geom
    summ = oracle.page_summaries(g, case.k_cache, case.page_table, case.seq_lens)
    sc = oracle.page_scores(g, case.q, summ, case.page_table, case.seq_lens)
    o_sel, o_cnt = oracle.select_pages(g, sc, case.seq_lens, case.budget, case.sink,
                                       case.window)
    assert np.array_equal(res["cnt"], o_cnt)
    assert np.array_equal(res["sel"], o_sel)
    fin = np.isfinite(sc)
    assert np.array_equal(res["scores"][fin], sc[fin].astype(np.float32))
    full_parity(case, res)


@pytest.mark.parametrize("kw", [dict(wl="tiny", B=3, seq_lens=[4096, 700, 0], Hkv=2, Hq=8),
                                dict(wl="llama32k", B=2, L=(3000, 9000), seed=71),
                                dict(wl="tiny", B=2, seq_lens=[5000, 33], Hkv=1, Hq=6, P=64,
                                     budget=1024, sink=64, window=256)])
def test_page_scores_alone(kw):
    kw = dict(kw)
    case = synth.decode_case(kw.pop("wl"), **kw)
    dc = DevCase(case)
    g = dc.g
    sa.page_summaries(g, dc.k, dc.pt, dc.sl, dc.summ)
    ws = sa.Workspace.for_decode(g, case.budget)
    sc = torch.full((g.B, g.Hkv, g.max_pages), 7.0, dtype=torch.float32, device="cuda")
    sa.page_scores(g, dc.q, dc.summ, dc.pt, dc.sl, ws, scores=sc)
    assert ws.status() == sa.SA_OK
    summ = oracle.page_summaries(case.geom, case.k_cache, case.page_table, case.seq_lens)
    ref = oracle.page_scores(case.geom, case.q, summ, case.page_table, case.seq_lens)
    got = sc.cpu().numpy()
    fin = np.isfinite(ref)
    assert np.array_equal(fin, np.isfinite(got))
    assert np.isneginf(got[~fin]).all()
    assert np.allclose(got[fin], ref[fin], rtol=1e-5, atol=1e-4)


# ------------------------------------------------------------------------------------
# latent (MLA) geometry: 128 query heads share one 576-wide latent key per token; the
# page scores run on the tcgen05 tensor cores
# ------------------------------------------------------------------------------------

MLA_CASES = [dict(B=2, L=(8192, 8192), seed=91),
             dict(B=3, seq_lens=[65536, 9000, 64], seed=92),
             dict(B=2, seq_lens=[0, 20000], seed=93, poison="nan")]


@pytest.mark.parametrize("kw", MLA_CASES, ids=lambda kw: "-".join(
    "%s%s" % (k, v if not isinstance(v, list) else len(v)) for k, v in kw.items()))
def test_mla_scores_and_selection(kw):
    case = synth.decode_case("mla", **kw)
    dc = DevCase(case)
    g = dc.g
    K = case.budget // g.P
    sa.page_summaries(g, dc.k, dc.pt, dc.sl, dc.summ)
    ws = sa.Workspace.for_decode(g, case.budget)
    sc = torch.full((g.B, g.Hkv, g.max_pages), 7.0, dtype=torch.float32, device="cuda")
    sa.page_scores(g, dc.q, dc.summ, dc.pt, dc.sl, ws, scores=sc)
    assert ws.status() == sa.SA_OK
    summ = oracle.page_summaries(case.geom, case.k_cache, case.page_table, case.seq_lens)
    assert np.array_equal(u16(dc.summ), summ)
    ref = oracle.page_scores(case.geom, case.q, summ, case.page_table, case.seq_lens)
    got = sc.cpu().numpy()
    fin = np.isfinite(ref)
    assert np.array_equal(fin, np.isfinite(got))
    assert np.allclose(got[fin], ref[fin], rtol=1e-5, atol=1e-3), \
        np.abs(got[fin] - ref[fin]).max()
    # selection through the C ABI, with the newest page refreshed first
    sel = torch.empty((g.B, g.Hkv, K), dtype=torch.int32, device="cuda")
    cnt = torch.empty((g.B, g.Hkv), dtype=torch.int32, device="cuda")
    phys = torch.empty_like(sel)
    sc2 = torch.empty_like(sc)
    sa.select_pages(g, dc.q, dc.summ, dc.pt, dc.sl, case.budget, case.sink, case.window, ws,
                    sel=sel, sel_count=cnt, scores=sc2, k_cache=dc.k, n_tail_refresh=1,
                    sel_phys=phys)
    assert ws.status() == sa.SA_OK
    assert np.array_equal(u16(dc.summ), summ)
    osel, ocnt = oracle.select_pages(case.geom, ref, case.seq_lens, case.budget, case.sink,
                                     case.window)
    from parity import check_selection
    check_selection(case.geom, case.seq_lens, case.budget, case.sink, case.window, ref, osel,
                    ocnt, sel.cpu().numpy(), cnt.cpu().numpy())
    gs, gc, gp = sel.cpu().numpy(), cnt.cpu().numpy(), phys.cpu().numpy()
    for b in range(g.B):
        c = gc[b, 0]
        assert np.array_equal(gp[b, 0, :c], case.page_table[b, gs[b, 0, :c]])


@pytest.mark.parametrize("kw", MLA_CASES + [dict(B=2, seq_lens=[65536, 4000], seed=94,
                                                  budget=4096, sink=64, window=1024)],
                         ids=lambda kw: "-".join("%s%s" % (k, v if not isinstance(v, list)
                                                           else len(v)) for k, v in kw.items()))
def test_mla_decode_parity(kw):
    # scores + selection + tensor-core attention over the latent rows (V = first 512)
    case = synth.decode_case("mla", **kw)
    res = run_decode(DevCase(case))
    full_parity(case, res)


def test_mla_deterministic_bitwise():
    case = synth.decode_case("mla", B=2, seq_lens=[30000, 9000], seed=96)
    dc = DevCase(case)
    a = run_decode(dc)
    b = run_decode(dc)
    for k in ("summ", "sel", "cnt", "out", "lse", "scores"):
        assert np.array_equal(a[k], b[k]), k


def test_sparse_decode_in_cuda_graph_replays():
    # captured once, replayed on new queries: the outputs follow the queries exactly
    case = synth.decode_case("llama32k", B=2, L=(8192, 8192), seed=97)
    dc = DevCase(case)
    g = dc.g
    sa.page_summaries(g, dc.k, dc.pt, dc.sl, dc.summ)
    ws = sa.Workspace.for_decode(g, case.budget)
    out = torch.empty((g.B, g.Hq, g.Dv), dtype=torch.float32, device="cuda")
    lse = torch.empty((g.B, g.Hq), dtype=torch.float32, device="cuda")
    q = dc.q.clone()
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        sa.sparse_decode(g, q, dc.k, dc.v, dc.summ, dc.pt, dc.sl, case.budget, case.sink,
                         case.window, case.scale, ws, out=out, lse=lse, stream=stream)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            sa.sparse_decode(g, q, dc.k, dc.v, dc.summ, dc.pt, dc.sl, case.budget, case.sink,
                             case.window, case.scale, ws, out=out, lse=lse, stream=stream)
    rng = np.random.default_rng(97)
    for _ in range(2):
        qn = synth.f32_to_bf16(rng.standard_normal(case.q.shape).astype(np.float32))
        q.copy_(to_dev(qn))
        with torch.cuda.stream(stream):
            graph.replay()
        torch.cuda.synchronize()
        assert ws.status() == sa.SA_OK
        c2 = dataclasses.replace(case, q=qn)
        res = dict(summ=u16(dc.summ), out=out.cpu().numpy(), lse=lse.cpu().numpy())
        ref_out, ref_lse = sa.sparse_decode(g, q, dc.k, dc.v, dc.summ, dc.pt, dc.sl, case.budget,
                                            case.sink, case.window, case.scale, ws)
        assert np.array_equal(res["out"], ref_out.cpu().numpy())
        assert np.array_equal(res["lse"], ref_lse.cpu().numpy())
        sc = oracle.page_scores(c2.geom, c2.q, oracle.page_summaries(c2.geom, c2.k_cache,
                                                                     c2.page_table, c2.seq_lens),
                                c2.page_table, c2.seq_lens)
        osel, ocnt = oracle.select_pages(c2.geom, sc, c2.seq_lens, c2.budget, c2.sink, c2.window)
        o, l = oracle.attend(c2.geom, c2.q, c2.k_cache, c2.v_cache, c2.page_table, c2.seq_lens,
                             osel, ocnt, c2.scale)
        check_attention(res["out"], res["lse"], o, l)


def test_mla_budget_covers_all_pages_equals_dense():
    case = synth.decode_case("mla", B=2, seq_lens=[1500, 777], budget=1536, seed=95)
    res = run_decode(DevCase(case))
    g = case.geom
    for b in range(g.B):
        L = int(case.seq_lens[b])
        rows = np.concatenate([case.k_cache[case.page_table[b, p], 0]
                               for p in range((L + g.P - 1) // g.P)])[:L]
        o, l = oracle.dense_attend(case.q[b], rows, rows[:, :g.Dv], case.scale)
        check_attention(res["out"][b], res["lse"][b], o, l)


def test_budget_covers_all_pages_equals_dense():
    case = synth.decode_case("tiny", B=2, seq_lens=[1234, 4096], Hkv=2, Hq=8, budget=4096,
                             poison="nan")
    res = run_decode(DevCase(case))
    g = case.geom
    for b in range(g.B):
        L = int(case.seq_lens[b])
        for h in range(g.Hkv):
            ks = np.concatenate([case.k_cache[case.page_table[b, p], h]
                                 for p in range((L + 15) // 16)])[:L]
            vs = np.concatenate([case.v_cache[case.page_table[b, p], h]
                                 for p in range((L + 15) // 16)])[:L]
            o, l = oracle.dense_attend(case.q[b, h * g.G:(h + 1) * g.G], ks, vs, case.scale)
            check_attention(res["out"][b, h * g.G:(h + 1) * g.G], res["lse"][b, h * g.G:(h + 1) * g.G],
                            o, l)


def test_empty_sequence_outputs():
    case = synth.decode_case("tiny", B=2, seq_lens=[0, 300], Hkv=1, Hq=4)
    res = run_decode(DevCase(case))
    assert (res["out"][0] == 0).all() and np.isneginf(res["lse"][0]).all()
    assert res["cnt"][0, 0] == 0 and (res["sel"][0, 0] == -1).all()
    full_parity(case, res)


def test_attend_selected_reuses_indices():
    # one layer's selection reused at another layer (different q, K, V; same lengths)
    c1 = synth.decode_case("llama32k", B=2, L=(4096, 4096), seed=31)
    c2 = synth.decode_case("llama32k", B=2, L=(4096, 4096), seed=32)
    d1, d2 = DevCase(c1), DevCase(c2)
    r1 = run_decode(d1, scores=False)
    ws = sa.Workspace.for_decode(d2.g, c2.budget)
    sel = to_dev(r1["sel"])
    cnt = to_dev(r1["cnt"])
    out, lse = sa.attend_selected(d2.g, d2.q, d2.k, d2.v, d2.pt, d2.sl, sel, cnt, c2.scale, ws)
    assert ws.status() == sa.SA_OK
    ro, rl = oracle.attend(c2.geom, c2.q, c2.k_cache, c2.v_cache, c2.page_table, c2.seq_lens,
                           r1["sel"], r1["cnt"], c2.scale)
    check_attention(out.cpu().numpy(), lse.cpu().numpy(), ro, rl)


# ------------------------------------------------------------------------------------
# fp8 summaries rounded outward: records bit-exact, scores and decode against the oracle
# ------------------------------------------------------------------------------------

FP8 = [
    dict(wl="tiny", B=3, seq_lens=[4096, 700, 33], Hkv=2, Hq=8, poison="nan"),
    dict(wl="tiny", B=2, seq_lens=[3000, 1], Hkv=4, Hq=32),
    dict(wl="llama32k", B=2, L=(8192, 8192), seed=91),
    dict(wl="ragged", B=2, L=(3000, 9000), seed=92, budget=1024, sink=128, window=256,
         poison="nan"),
]


def _fp8_check(case, dc, s8, lse_rel=None):
    g = dc.g
    ref8 = oracle.page_summaries_fp8(case.geom, case.k_cache, case.page_table, case.seq_lens)
    assert np.array_equal(s8.cpu().numpy(), ref8)
    osc = oracle.page_scores_fp8(case.geom, case.q, ref8, case.page_table, case.seq_lens)
    ws = sa.Workspace.for_decode(g, case.budget)
    gsc = sa.page_scores_fp8(g, dc.q, s8, dc.pt, dc.sl, ws).cpu().numpy()
    fin = np.isfinite(osc)
    assert np.array_equal(fin, np.isfinite(gsc))
    assert np.allclose(gsc[fin], osc[fin], rtol=1e-5, atol=1e-4)
    K = case.budget // g.P
    sel = torch.empty((g.B, g.Hkv, K), dtype=torch.int32, device="cuda")
    cnt = torch.empty((g.B, g.Hkv), dtype=torch.int32, device="cuda")
    out, lse = sa.sparse_decode_fp8(g, dc.q, dc.k, dc.v, s8, dc.pt, dc.sl, case.budget,
                                    case.sink, case.window, case.scale, ws, sel_out=sel,
                                    sel_count_out=cnt)
    assert ws.status() == sa.SA_OK
    gs, gc = sel.cpu().numpy(), cnt.cpu().numpy()
    osel, ocnt = oracle.select_pages(case.geom, osc, case.seq_lens, case.budget, case.sink,
                                     case.window)
    tied = check_selection(case.geom, case.seq_lens, case.budget, case.sink, case.window, osc,
                           osel, ocnt, gs, gc)
    o, l = oracle.attend(case.geom, case.q, case.k_cache, case.v_cache, case.page_table,
                         case.seq_lens, gs if tied else osel, ocnt, case.scale)
    if lse_rel is None:
        check_attention(out.cpu().numpy(), lse.cpu().numpy(), o, l)
    else:
        # logits far beyond 1e3: lse to fp32 relative accuracy, out as usual
        gl = lse.cpu().numpy()
        check_attention(out.cpu().numpy(), l, o, l)
        assert np.array_equal(np.isfinite(gl), np.isfinite(l))
        f = np.isfinite(l)
        assert (np.abs(gl[f] - l[f]) <= lse_rel * np.abs(l[f]) + 1e-3).all()
    return gsc


@pytest.mark.parametrize("kw", FP8, ids=lambda kw: "%s-B%d" % (kw["wl"], kw["B"]))
def test_fp8_summaries_scores_and_decode(kw):
    kw = dict(kw)
    case = synth.decode_case(kw.pop("wl"), **kw)
    dc = DevCase(case)
    g = dc.g
    s8 = sa.empty_summaries_fp8(g)
    sa.page_summaries_fp8(g, dc.k, dc.pt, dc.sl, s8)
    gsc = _fp8_check(case, dc, s8)
    # never below the bf16 bound of the same pages
    sa.page_summaries(g, dc.k, dc.pt, dc.sl, dc.summ)
    ws = sa.Workspace.for_decode(g, case.budget)
    s16 = sa.page_scores(g, dc.q, dc.summ, dc.pt, dc.sl, ws).cpu().numpy()
    fin = np.isfinite(s16)
    assert (gsc[fin] >= s16[fin] - 1e-5 * np.abs(s16[fin]) - 1e-4).all()


def test_fp8_records_extreme_magnitudes():
    # pages scaled by powers of two from 2^-40 to 2^60: positive and negative record
    # exponents, E4M3 subnormals, and codes at 448
    case = synth.decode_case("tiny", B=2, seq_lens=[1600, 900], Hkv=2, Hq=8, seed=93)
    k = synth.bf16_to_f32(case.k_cache).astype(np.float64)
    pw = np.array([-40, -12, -3, 0, 5, 20, 60])
    s = pw[np.arange(k.shape[0]) % len(pw)]
    k = k * (2.0 ** s)[:, None, None, None]
    k[0::5, :, :, 7] = 0.0           # all-zero channels
    k[1::9] = 0.0                    # all-zero pages: e = 0
    case = dataclasses.replace(case, k_cache=synth.f32_to_bf16(k.astype(np.float32)))
    dc = DevCase(case)
    s8 = sa.empty_summaries_fp8(dc.g)
    sa.page_summaries_fp8(dc.g, dc.k, dc.pt, dc.sl, s8)
    _fp8_check(case, dc, s8, lse_rel=1e-5)


def test_fp8_tail_refresh_inside_decode():
    case = synth.decode_case("llama32k", B=3, seq_lens=[4097, 3000, 2064], seed=94,
                             poison="nan")
    dc = DevCase(case)
    g = dc.g
    before = to_dev(np.maximum(case.seq_lens - 1, 0))
    s8 = sa.empty_summaries_fp8(g)
    sa.page_summaries_fp8(g, dc.k, dc.pt, before, s8)      # newest page stale
    ws = sa.Workspace.for_decode(g, case.budget)
    out, lse = sa.sparse_decode_fp8(g, dc.q, dc.k, dc.v, s8, dc.pt, dc.sl, case.budget,
                                    case.sink, case.window, case.scale, ws, n_tail_refresh=1)
    assert ws.status() == sa.SA_OK
    ref = oracle.decode_fp8(case)
    assert np.array_equal(s8.cpu().numpy(), ref["summ8"])
    check_attention(out.cpu().numpy(), lse.cpu().numpy(), ref["out"], ref["lse"])
    # update_summaries_fp8 alone gives the same records
    s8b = sa.empty_summaries_fp8(g)
    sa.page_summaries_fp8(g, dc.k, dc.pt, before, s8b)
    sa.update_summaries_fp8(g, dc.k, dc.pt, dc.sl, s8b, n_tail_pages=1)
    assert np.array_equal(s8b.cpu().numpy(), ref["summ8"])


def test_fp8_rejects_the_latent_geometry():
    case = synth.decode_case("mla", B=1, seq_lens=[640])
    g = sa.Geometry.of(case.geom)
    assert sa.summary_fp8_record_bytes(g) == 0
    with pytest.raises(sa.SaError):
        sa.empty_summaries_fp8(g)


def test_cross_layer_reuse_of_physical_pages():
    # layer 0 selects and returns the physical pages of its selection; the next layer
    # (own q, K, V; the same page table and lengths) attends over those physical pages
    lens = [4096, 1000, 2500]
    c0 = synth.decode_case("llama32k", B=3, seq_lens=lens, seed=41)
    other = synth.decode_case("llama32k", B=3, seq_lens=lens, seed=42)
    assert other.k_cache.shape == c0.k_cache.shape
    c1 = dataclasses.replace(c0, q=other.q, k_cache=other.k_cache, v_cache=other.v_cache)
    d0, d1 = DevCase(c0), DevCase(c1)
    g = d0.g
    K = c0.budget // g.P
    ws = sa.Workspace.for_decode(g, c0.budget)
    sa.page_summaries(g, d0.k, d0.pt, d0.sl, d0.summ)
    sel = torch.empty((g.B, g.Hkv, K), dtype=torch.int32, device="cuda")
    cnt = torch.empty((g.B, g.Hkv), dtype=torch.int32, device="cuda")
    phys = torch.empty_like(sel)
    sa.select_pages(g, d0.q, d0.summ, d0.pt, d0.sl, c0.budget, c0.sink, c0.window, ws,
                    sel=sel, sel_count=cnt, sel_phys=phys)
    out, lse = sa.attend_selected(g, d1.q, d1.k, d1.v, d1.pt, d1.sl, sel, cnt, c1.scale, ws,
                                  sel_phys=phys)
    assert ws.status() == sa.SA_OK
    gs, gc = sel.cpu().numpy(), cnt.cpu().numpy()
    summ = oracle.page_summaries(c0.geom, c0.k_cache, c0.page_table, c0.seq_lens)
    sc = oracle.page_scores(c0.geom, c0.q, summ, c0.page_table, c0.seq_lens)
    osel, ocnt = oracle.select_pages(c0.geom, sc, c0.seq_lens, c0.budget, c0.sink, c0.window)
    tied = check_selection(c0.geom, c0.seq_lens, c0.budget, c0.sink, c0.window, sc, osel, ocnt,
                           gs, gc)
    ro, rl = oracle.attend(c1.geom, c1.q, c1.k_cache, c1.v_cache, c1.page_table, c1.seq_lens,
                           gs if tied else osel, ocnt, c1.scale)
    check_attention(out.cpu().numpy(), lse.cpu().numpy(), ro, rl)
    # the same outputs as when layer 1 looks its pages up through the page table itself
    out2, lse2 = sa.attend_selected(g, d1.q, d1.k, d1.v, d1.pt, d1.sl, sel, cnt, c1.scale, ws)
    assert np.array_equal(out2.cpu().numpy(), out.cpu().numpy())
    assert np.array_equal(lse2.cpu().numpy(), lse.cpu().numpy())


def test_deterministic_bitwise():
    case = synth.decode_case("llama32k", B=2, L=(8192, 8192), seed=17)
    dc = DevCase(case)
    a = run_decode(dc)
    b = run_decode(dc)
    for k in ("summ", "sel", "cnt", "out", "lse", "scores"):
        assert np.array_equal(a[k], b[k]), k


# ------------------------------------------------------------------------------------
# invalid arguments are rejected on the host before any launch
# ------------------------------------------------------------------------------------

def test_invalid_arguments():
    case = synth.decode_case("tiny")
    dc = DevCase(case)
    g = dc.g
    ws = sa.Workspace.for_decode(g, case.budget)
    with pytest.raises(sa.SaError) as e:
        sa.sparse_decode(g, dc.q, dc.k, dc.v, dc.summ, dc.pt, dc.sl, case.budget, 512, 64,
                         case.scale, ws)
    assert e.value.status == -1                        # sink + window > budget
    with pytest.raises(sa.SaError) as e:
        sa.sparse_decode(g, dc.q, dc.k, dc.v, dc.summ, dc.pt, dc.sl, 500, 16, 64, case.scale, ws)
    assert e.value.status == -1                        # budget not a multiple of P
    small = sa.Workspace(256)
    with pytest.raises(sa.SaError) as e:
        sa.sparse_decode(g, dc.q, dc.k, dc.v, dc.summ, dc.pt, dc.sl, case.budget, 16, 64,
                         case.scale, small)
    assert e.value.status == -3                        # workspace too small
    bad = dataclasses.replace(g, Dk=96, Dv=96)
    with pytest.raises(sa.SaError) as e:
        sa.page_summaries(bad, dc.k, dc.pt, dc.sl, dc.summ)
    assert e.value.status == -2                        # unsupported head dim
    bad = dataclasses.replace(g, Hq=5, Hkv=2)
    with pytest.raises(sa.SaError) as e:
        sa.page_summaries(bad, dc.k, dc.pt, dc.sl, dc.summ)
    assert e.value.status == -1                        # Hq % Hkv != 0
    assert ws.status() == sa.SA_OK


# ------------------------------------------------------------------------------------
# prefix-cache pruning (bit-exact)
# ------------------------------------------------------------------------------------

def _run_prune(pc, n_free=None):
    d = pc.decode
    g = sa.Geometry.of(d.geom)
    k, v = to_dev(d.k_cache), to_dev(d.v_cache) if d.v_cache is not None else None
    summ = torch.zeros((g.n_pool, g.Hkv, 2, g.Dk), dtype=torch.int16, device="cuda")
    ws = sa.Workspace.for_prune(g)
    fp = to_dev(pc.free_pages if n_free is None else pc.free_pages[:n_free])
    npt, nsl, pos, ll = sa.prune_compact(g, k, v, to_dev(d.page_table), to_dev(d.seq_lens),
                                         to_dev(pc.keep), fp, k, v, summ, ws)
    st = ws.status()
    return st, dict(k_dst=u16(k), v_dst=u16(v) if v is not None else None, summ=u16(summ),
                    new_page_table=npt.cpu().numpy(), new_seq_lens=nsl.cpu().numpy(),
                    pos_map=pos.cpu().numpy(), logical_len=ll.cpu().numpy())


@pytest.mark.parametrize("kw", [
    dict(B=3, seq_lens=[3000, 2200, 5000], Hkv=2, Hq=8),
    dict(B=4, seq_lens=[0, 1, 17, 9000], Hkv=8, Hq=32, extra_free=5),
    dict(B=2, seq_lens=[4100, 300], Hkv=8, Hq=32, P=32),
    dict(B=2, seq_lens=[8200, 100], Hkv=4, Hq=8, P=64),
    dict(B=2, seq_lens=[3000, 700], Hkv=2, Hq=8, keep_all=True),
    dict(B=2, seq_lens=[3000, 700], Hkv=2, Hq=8, keep_none=True),
])
def test_prune_bit_exact(kw):
    pc = synth.prune_case("prune", **kw)
    st, r = _run_prune(pc)
    assert st == sa.SA_OK
    d = pc.decode
    ref = oracle.prune_compact(d.geom, d.k_cache, d.v_cache, d.page_table, d.seq_lens, pc.keep,
                               pc.free_pages)
    summ_ref = ref["summ"]
    for key in ("new_page_table", "new_seq_lens", "pos_map", "logical_len", "k_dst", "v_dst"):
        assert np.array_equal(r[key], ref[key]), key
    # the oracle writes summaries of new pages only; so does the library
    assert np.array_equal(r["summ"], summ_ref)


def test_prune_latent_pool():
    pc = synth.prune_case("mla", B=2, seq_lens=[3000, 640], Hq=128, budget=640, sink=64,
                          window=128)
    st, r = _run_prune(pc)
    assert st == sa.SA_OK
    d = pc.decode
    ref = oracle.prune_compact(d.geom, d.k_cache, None, d.page_table, d.seq_lens, pc.keep,
                               pc.free_pages)
    for key in ("new_page_table", "new_seq_lens", "pos_map", "logical_len", "k_dst", "summ"):
        assert np.array_equal(r[key], ref[key]), key


def test_prune_reports_no_space_and_writes_nothing():
    pc = synth.prune_case("prune", B=2, seq_lens=[3000, 2200], Hkv=2, Hq=8)
    d = pc.decode
    st, r = _run_prune(pc, n_free=len(pc.free_pages) - 1)
    assert st == -7                                    # SA_ERR_NO_SPACE
    assert np.array_equal(r["k_dst"], d.k_cache)       # pool untouched
    assert (r["summ"] == 0).all()


def test_decode_after_prune():
    pc = synth.prune_case("prune", B=3, seq_lens=[9000, 12000, 5000], Hkv=8, Hq=32)
    st, r = _run_prune(pc)
    assert st == sa.SA_OK
    d = pc.decode
    comp = dataclasses.replace(d, k_cache=r["k_dst"], v_cache=r["v_dst"],
                               page_table=r["new_page_table"], seq_lens=r["new_seq_lens"])
    res = run_decode(DevCase(comp))
    full_parity(comp, res)
