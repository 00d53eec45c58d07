"""sa_sparse_decode_noalloc: the workspace-free variant of sa_sparse_decode.

Runs last in the suite (file name) and also passes on its own: the library's static
scratch must give the same results as a caller-owned workspace on consecutive calls,
and geometries whose workspace exceeds the scratch are refused before any launch.
"""

import numpy as np
import pytest

import oracle
import synth
from parity import DevCase, check_attention, check_selection

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import paged_kv_cache_sa_b200 as sa  # noqa: E402


@pytest.mark.parametrize("kw", [dict(wl="llama32k", B=2, L=(8192, 8192), seed=81),
                                dict(wl="tiny", B=3, seq_lens=[4096, 700, 0], Hkv=2, Hq=8,
                                     seed=82),
                                # latent geometry small enough for the static scratch
                                dict(wl="mla", B=2, L=(8192, 8192), seed=83)])
def test_noalloc_matches_workspace_decode_on_consecutive_calls(kw):
    kw = dict(kw)
    case = synth.decode_case(kw.pop("wl"), **kw)
    dc = DevCase(case)
    g = dc.g
    K = case.budget // g.P
    assert sa.decode_workspace_size(g, case.budget) <= 32 << 20
    sa.page_summaries(g, dc.k, dc.pt, dc.sl, dc.summ)
    ws = sa.Workspace.for_decode(g, case.budget)
    sel_r = torch.empty((g.B, g.Hkv, K), dtype=torch.int32, device="cuda")
    cnt_r = torch.empty((g.B, g.Hkv), dtype=torch.int32, device="cuda")
    out_r, lse_r = sa.sparse_decode(g, dc.q, dc.k, dc.v, dc.summ, dc.pt, dc.sl, case.budget,
                                    case.sink, case.window, case.scale, ws, sel_out=sel_r,
                                    sel_count_out=cnt_r, n_tail_refresh=1)
    assert ws.status() == sa.SA_OK
    ref = (out_r.cpu().numpy(), lse_r.cpu().numpy(), sel_r.cpu().numpy(), cnt_r.cpu().numpy())
    for _ in range(2):
        sel = torch.full((g.B, g.Hkv, K), 123, dtype=torch.int32, device="cuda")
        cnt = torch.full((g.B, g.Hkv), 123, dtype=torch.int32, device="cuda")
        st = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        out, lse = sa.sparse_decode_noalloc(g, dc.q, dc.k, dc.v, dc.summ, dc.pt, dc.sl,
                                            case.budget, case.sink, case.window, case.scale,
                                            sel_out=sel, sel_count_out=cnt, status_out=st,
                                            n_tail_refresh=1)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        assert np.array_equal(sel.cpu().numpy(), ref[2])
        assert np.array_equal(cnt.cpu().numpy(), ref[3])
        check_attention(out.cpu().numpy(), lse.cpu().numpy(), ref[0], ref[1])
    # and against the oracle: the selection bit-exact outside the tie band, the attention
    # over the selection made within the stated tolerance
    o = oracle.decode(case)
    check_selection(case.geom, case.seq_lens, case.budget, case.sink, case.window,
                    o["scores"], o["sel"], o["sel_count"], ref[2], ref[3])
    oa = oracle.decode(case, sel=ref[2], sel_count=ref[3])
    check_attention(out.cpu().numpy(), lse.cpu().numpy(), oa["out"], oa["lse"])


def test_noalloc_refuses_workspace_above_the_scratch():
    # scores alone need B * Hkv * max_pages * 4 = 64 MiB > SA_STATIC_SCRATCH_BYTES
    g = sa.Geometry(B=64, Hq=32, Hkv=8, Dk=128, Dv=128, P=16, max_pages=32768, n_pool=1024)
    assert sa.decode_workspace_size(g, 2048) > 32 << 20
    q = torch.zeros((64, 32, 128), dtype=torch.int16, device="cuda")
    kv = torch.zeros((1024, 8, 16, 128), dtype=torch.int16, device="cuda")
    summ = torch.zeros((1024, 8, 2, 128), dtype=torch.int16, device="cuda")
    pt = torch.zeros((64, 32768), dtype=torch.int32, device="cuda")
    sl = torch.zeros((64,), dtype=torch.int32, device="cuda")
    with pytest.raises(sa.SaError) as e:
        sa.sparse_decode_noalloc(g, q, kv, kv, summ, pt, sl, 2048, 64, 512, 0.088)
    assert e.value.status == sa.SA_ERR_WORKSPACE
